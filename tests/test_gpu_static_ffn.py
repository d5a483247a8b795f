"""FFN with a static neuron mask on both projections vs the oracle (GPU).

"GLASS: Global-Local Aggregation for inference-time Sparsification",
"selection": the prompt-fixed neuron set skips the pruned neurons' up columns
and down rows. The oracle writes the dense definition (act(x W_a) then
(h * m) W_d); the GPU reads only the kept rows of the [ffn x d] matrices.
"""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import assert_close, to64
from sparse_input_gemv_b200 import binding as sb
from sparse_input_gemv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sb.load()


def dev(t):
    return t.to("cuda").contiguous()


def make(name, B, d, ffn, dtype, swiglu):
    Wa = synth.normal((d, ffn), synth.seed_of(name, "Wa"), 0.02, dtype)
    Wb = synth.normal((d, ffn), synth.seed_of(name, "Wb"), 0.02, dtype) if swiglu else None
    Wd = synth.normal((ffn, d), synth.seed_of(name, "Wd"), 0.02, dtype)
    x = synth.eval_draw(name, "x", B, d, dtype)
    return x, Wa, Wb, Wd


def run(name, B, d, ffn, keep_idx, dtype="bf16", act="gelu", ws=None):
    swiglu = act == "swiglu"
    x, Wa, Wb, Wd = make(name, B, d, ffn, dtype, swiglu)
    idx = torch.as_tensor(np.asarray(keep_idx, dtype=np.int32))
    cnt = torch.tensor([idx.numel()], dtype=torch.int32)
    flags = sb.SFX_FLAG_GELU_TANH if act == "gelu_tanh" else 0
    y = sb.sfx_static_ffn(dev(x), dev(Wa.t()), dev(Wd), dev(idx) if idx.numel() else
                          torch.zeros(1, dtype=torch.int32, device="cuda"), dev(cnt),
                          W_bT=dev(Wb.t()) if swiglu else None, flags=flags,
                          out_dtype=torch.float32, ws=ws)
    keep = np.zeros(ffn, bool)
    keep[np.asarray(keep_idx, dtype=np.int64)] = True
    want, _ = O.ffn_static_mask(to64(x), to64(Wa), to64(Wd), keep, act=act,
                                W_b=to64(Wb) if swiglu else None)
    return to64(y), want


@pytest.mark.parametrize("B", [1, 3, 16])
@pytest.mark.parametrize("act", ["gelu", "gelu_tanh", "swiglu"])
def test_static_ffn_small_ragged(B, act):
    d, ffn = 264, 200
    rng = np.random.default_rng(7)
    keep = np.sort(rng.choice(ffn, size=83, replace=False))
    y, want = run("static-small", B, d, ffn, keep, act=act)
    assert_close(y, O.round_to(want, "f32"), f"static {act} B={B}")


def test_static_ffn_any_order_all_and_one():
    d, ffn = 256, 130
    rng = np.random.default_rng(9)
    keep = rng.permutation(ffn)  # every neuron, unsorted: the dense FFN
    y, want = run("static-all", 2, d, ffn, keep, act="swiglu")
    assert_close(y, O.round_to(want, "f32"), "all kept")
    y1, want1 = run("static-one", 2, d, ffn, [77], act="gelu")
    assert_close(y1, O.round_to(want1, "f32"), "one kept")


def test_static_ffn_empty_set_gives_zero():
    y, want = run("static-none", 4, 128, 64, [], act="gelu")
    assert np.all(want == 0.0)
    assert np.all(y == 0.0)


def test_static_ffn_phi2_with_glass_set():
    # Phi-2-shaped GeLU FFN, fp16, with the neuron set of a GLASS selection
    d, ffn, keep = 2560, 10240, 0.3
    k = O.keep_count(keep, ffn)
    sl = synth.abs_normal((1, ffn), synth.seed_of("static-phi2", "local"))
    sg = synth.abs_normal((1, ffn), synth.seed_of("static-phi2", "global"))
    sel = sb.sfx_mask_compact(None, sb.SFX_SEL_TOPK_GLASS, k=k, score_l=dev(sl), score_g=dev(sg),
                              lam=0.5)
    want_mask = O.glass_mask(sl.numpy()[0], sg.numpy()[0], 0.5, k)
    idx = sel["idx"][0, :k].cpu().numpy()
    assert np.array_equal(idx, O.compact(want_mask)[0])
    y, want = run("static-phi2", 1, d, ffn, idx, dtype="f16", act="gelu")
    assert_close(y, O.round_to(want, "f32"), "phi2 glass")


def test_static_ffn_llama3_8b_swiglu_half_kept():
    d, ffn = 4096, 14336
    rng = np.random.default_rng(13)
    keep = np.sort(rng.choice(ffn, size=ffn // 2, replace=False))
    y, want = run("static-8b", 4, d, ffn, keep, dtype="bf16", act="swiglu")
    assert_close(y, O.round_to(want, "f32"), "8b swiglu")


def test_static_ffn_bad_index_is_skipped_and_flagged():
    d, ffn = 256, 96
    ws = sb.Workspace()
    x, Wa, _, Wd = make("static-bad", 1, d, ffn, "bf16", False)
    idx = torch.tensor([5, ffn + 3, 40, -1], dtype=torch.int32)
    cnt = torch.tensor([4], dtype=torch.int32)
    y = sb.sfx_static_ffn(dev(x), dev(Wa.t()), dev(Wd), dev(idx), dev(cnt),
                          out_dtype=torch.float32, ws=ws)
    assert ws.status() == sb.SFX_DEV_BAD_INDEX
    keep = np.zeros(ffn, bool)
    keep[[5, 40]] = True
    want, _ = O.ffn_static_mask(to64(x), to64(Wa), to64(Wd), keep)
    assert_close(to64(y), O.round_to(want, "f32"), "bad idx")
