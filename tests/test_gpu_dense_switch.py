"""The sparse/dense switch of the batch path and its dense kernel (GPU).

"Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
Model Execution", method: sparse execution pays off for small batches, and a
dense execution takes over when the batch grows. Here a batch of 3-16 tokens
runs either the union kernels (the rows any token keeps, gathered) or the
dense kernel (every row streamed as 2-D TMA tiles, multiplied by mma.sync
warps; a tcgen05 version is kept for comparison), chosen
on the device from the union's row count; rows no token keeps multiply zeros,
so both compute the same masked product. Each path is forced here and
compared with the fp64 oracle; the automatic choice is checked on either side
of the switch point.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from helpers import assert_close, pack_bitmap, to64
from sparse_input_gemv_b200 import binding as sb
from sparse_input_gemv_b200 import synth

pytestmark = pytest.mark.gpu

DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sb.load()
    yield
    ws = sb.default_workspace()
    if ws.buf is not None:
        assert ws.status() == 0, "device status word raised"


def dev(t):
    return t.to("cuda").contiguous()


def case(B, K, N, p, wdt="bf16", xdt=None, out="f32", flags=0, seed="dense", corr=False):
    xdt = xdt or wdt
    if corr:
        calib = synth.correlated_draws(seed, f"in{K}", 64, K, xdt, draw=0)
        x = synth.correlated_draws(seed, f"in{K}", B, K, xdt)
    else:
        calib = synth.calib_draws(seed, f"in{K}", 64, K, xdt)
        x = synth.eval_draw(seed, f"in{K}", B, K, xdt)
    t = O.calibrate_threshold(to64(calib), p) if p > 0 else -math.inf
    W = synth.normal((K, N), synth.seed_of(seed, K, N, "W"), 0.02, wdt)
    y, bm = sb.sfx_sparse_gemv(dev(x), dev(W), t=t, out_dtype=DT[out], flags=flags,
                               want_bitmap=True)
    m = O.magnitude_mask(to64(x), t)
    assert np.array_equal(bm.cpu().numpy(), pack_bitmap(m)), "fused mask differs"
    if flags & sb.SFX_FLAG_UNION_MASK:
        m = np.broadcast_to(O.union_mask(m), m.shape)
    want = O.masked_gemv(to64(x), m, to64(W))
    if flags & sb.SFX_FLAG_GELU:
        want = O.gelu_erf(want)
    if flags & sb.SFX_FLAG_SWIGLU:
        want = O.silu(want[:, 0::2]) * want[:, 1::2]
        out = "f32"
    assert_close(to64(y), O.round_to(want, out), f"B={B} K={K} N={N} p={p}")
    return y, O.union_mask(O.magnitude_mask(to64(x), t)).mean()


@pytest.mark.parametrize("B,K,N,p,wdt,xdt,out,flags", [
    (16, 4096, 2048, 0.5, "bf16", "bf16", "bf16", 0),
    (16, 8192, 2048, 0.0, "bf16", "bf16", "f32", 0),          # one tile split over ~9 CTAs
    (5, 1000, 264, 0.3, "f16", "f16", "f32", 0),              # ragged K and N (past-end boxes)
    (3, 33, 136, 0.0, "bf16", "bf16", "f32", 0),              # one partial stage
    (8, 14336, 4096, 0.65, "bf16", "f32", "bf16", 0),         # fp32 x: hi + lo tiles
    (11, 3000, 1000, 0.5, "f16", "f32", "f16", 0),
    (16, 256, 57344, 0.2, "bf16", "bf16", "f32", 0),          # many tiles, two stages each
    (9, 2048, 4096, 0.4, "bf16", "bf16", "f32", sb.SFX_FLAG_SWIGLU),
    (4, 2560, 1024, 0.4, "f16", "f16", "f32", sb.SFX_FLAG_GELU),
    (6, 1024, 512, 0.6, "bf16", "bf16", "f32", sb.SFX_FLAG_UNION_MASK),
])
@pytest.mark.parametrize("flavour", ["mma", "tcgen05"])
def test_dense_kernel_matches_oracle(B, K, N, p, wdt, xdt, out, flags, flavour):
    mode = sb.DENSE_ONLY if flavour == "mma" else sb.DENSE_ONLY_TCGEN05
    with sb.plan_overrides(dense=mode):
        case(B, K, N, p, wdt, xdt, out, flags, seed="dense-forced")


def test_dense_and_union_kernels_agree_at_full_size():
    # Llama-3-8B gate|up shape at 16 tokens, half the inputs masked
    B, K, N = 16, 4096, 28672
    x = dev(synth.eval_draw("dense-vs-union", "x", B, K, "bf16"))
    W = synth.normal((K, N), synth.seed_of("dense-vs-union", "W"), 0.02, "bf16", "cuda")
    t = 0.69
    with sb.plan_overrides(dense=sb.DENSE_ONLY):
        y_d = sb.sfx_sparse_gemv(x, W, t=t, out_dtype=torch.float32)
        y_d2 = sb.sfx_sparse_gemv(x, W, t=t, out_dtype=torch.float32)
    with sb.plan_overrides(dense=sb.DENSE_ONLY_TCGEN05):
        y_t = sb.sfx_sparse_gemv(x, W, t=t, out_dtype=torch.float32)
    with sb.plan_overrides(dense=sb.DENSE_UNION_ONLY):
        y_u = sb.sfx_sparse_gemv(x, W, t=t, out_dtype=torch.float32)
    assert torch.equal(y_d, y_d2), "the dense kernel adds its partials in a fixed order"
    # and both against the oracle on sampled columns
    cols = np.sort(np.random.default_rng(5).choice(N, size=512, replace=False))
    Wc = W[:, torch.from_numpy(cols).cuda()].double().cpu().numpy()
    x64 = to64(x)
    want = O.masked_gemv(x64, O.magnitude_mask(x64, t), Wc)
    assert_close(to64(y_d)[:, cols], O.round_to(want, "f32"), "dense kernel")
    assert_close(to64(y_u)[:, cols], O.round_to(want, "f32"), "union kernel")
    assert_close(to64(y_t)[:, cols], O.round_to(want, "f32"), "tcgen05 dense kernel")


@pytest.mark.parametrize("B,p,corr", [(16, 0.5, False), (16, 0.9, True), (4, 0.9, False)])
def test_switch_on_both_sides(B, p, corr):
    # iid tokens at p = 0.5: the union keeps ~all rows (dense side); correlated
    # tokens at p = 0.9 keep about a third (union side)
    y, union = case(B, 4096, 6144, p, corr=corr, seed="dense-auto")
    if corr:
        assert union < 0.5
    elif p == 0.5:
        assert union > 0.9
