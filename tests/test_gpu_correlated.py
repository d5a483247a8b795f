"""Batch-union kernels on correlated-token inputs, against the fp64 oracle.

The correlated recipe (``synth.correlated_draws``: per-neuron scales shared by
the tokens, so their masks overlap the way "GLASS: Global-Local Aggregation for
inference-time Sparsification" reports in its oracle-overlap analysis) makes
the batch union much sparser than iid draws do: at 16 tokens and p = 0.9 it
keeps about a third of the rows. These cases check the union path where it
really skips rows: the fused per-token masks bit for bit, the outputs within
the float tolerance, and the union actually below full density.
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


@pytest.mark.parametrize("B,p", [(4, 0.5), (4, 0.9), (16, 0.5), (16, 0.9)])
def test_union_gemv_correlated_tokens(B, p):
    K, N = 4096, 14336   # Llama-3-8B gate-shaped
    calib = synth.correlated_draws("corr-gemv", "x", 64, K, "bf16", draw=0)
    t = O.calibrate_threshold(to64(calib), p)
    x = synth.correlated_draws("corr-gemv", "x", B, K, "bf16")
    W = synth.normal((K, N), synth.seed_of("corr-gemv", "W"), 0.02, "bf16")
    assert sb.sfx_gemv_plan(B, K, N)["kernel"] == "union_mma"
    y, bm = sb.sfx_sparse_gemv(dev(x), dev(W), t=t, out_dtype=torch.float32, want_bitmap=True)
    m = O.magnitude_mask(to64(x), t)
    assert np.array_equal(bm.cpu().numpy(), pack_bitmap(m)), "fused mask differs"
    union = O.union_mask(m).mean()
    if p >= 0.9:
        assert union < 0.6, union   # the union really skips rows here
    want = O.masked_gemv(to64(x), m, to64(W))
    assert_close(to64(y), O.round_to(want, "f32"), f"B={B} p={p} union={union:.2f}")


@pytest.mark.parametrize("B,p", [(4, 0.5), (16, 0.9)])
def test_union_ffn_correlated_tokens(B, p):
    d, ffn = 4096, 14336
    calib = synth.correlated_draws("corr-ffn", "x", 64, d, "bf16", draw=0)
    t_in = O.calibrate_threshold(to64(calib), p)
    Wg = synth.normal((d, ffn), synth.seed_of("corr-ffn", "g"), 0.02, "bf16", "cuda")
    Wu = synth.normal((d, ffn), synth.seed_of("corr-ffn", "u"), 0.02, "bf16", "cuda")
    Wd = synth.normal((ffn, d), synth.seed_of("corr-ffn", "d"), 0.02, "bf16", "cuda")
    Wgu = sb.sfx_pack_gate_up(Wg, Wu)
    Wg64, Wu64, Wd64 = to64(Wg), to64(Wu), to64(Wd)
    _, hc, _, _ = O.ffn_swiglu(to64(calib[:16]), -math.inf, Wg64, Wu64, Wd64, -math.inf)
    t_h = float(np.float32(O.calibrate_threshold(hc, p)))
    x = synth.correlated_draws("corr-ffn", "x", B, d, "bf16")
    out = sb.sfx_sparse_ffn_swiglu(dev(x), Wgu, Wd, t_in, t_h, want_h=True, want_bitmaps=True)
    y, h, m_x, m_h = O.ffn_swiglu(to64(x), t_in, Wg64, Wu64, Wd64, t_h)
    assert np.array_equal(out["bitmap_x"].cpu().numpy(), pack_bitmap(m_x))
    assert_close(to64(out["h"]), O.round_to(h, "f32"), "h")
    # the down-site mask may differ only where fp32 and fp64 h straddle t_h
    got = np.unpackbits(out["bitmap_h"].cpu().numpy().view(np.uint8), bitorder="little")
    got = got.reshape(B, -1)[:, :ffn].astype(bool)
    flips = np.argwhere(got != m_h)
    for b, j in flips:
        assert abs(abs(h[b, j]) - t_h) <= 1e-4 * np.abs(h).max(), (b, j)
    assert len(flips) <= 2
    assert_close(to64(out["y"]), O.round_to(y, "bf16"), f"y B={B} p={p}")
