"""Batch-union product on mma.sync with register-direct weight loads (GPU).

"TEAL: Training-Free Activation Sparsity in Large Language Models", slides 8
and 19: each token keeps the rows with |x[b, i]| > t; a batch reads the union of
its tokens' rows once. Here the union GEMM kernel that loads weight rows
straight into registers and transposes them with movmatrix is selected for
every batch of 2 or more tokens, and compared with the fp64 oracle (rel-L2 <=
1e-3, max-abs <= 1e-2 max|y| of the oracle rounded to the output dtype) and
with the CUDA-core kernel.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from helpers import assert_close, pack_bitmap, to64
from sparse_input_gemv_b200 import binding as sb
from sparse_input_gemv_b200 import synth
from test_gpu_parity import ffn_case

pytestmark = pytest.mark.gpu

DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(autouse=True)
def _mma_union(monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sb.load()
    with sb.plan_overrides(union_kernel=sb.UNION_MMA, union_min_b=2):
        yield
    ws = sb.default_workspace()
    if ws.buf is not None:
        assert ws.status() == 0, "device status word raised"


def dev(t):
    return t.to("cuda").contiguous()


def case(B, K, N, p, wdt, xdt, out, flags=0, seed="mma"):
    calib = synth.calib_draws(seed, f"in{K}", 64, K, xdt)
    t = O.calibrate_threshold(to64(calib), p) if p > 0 else -math.inf
    x = synth.eval_draw(seed, f"in{K}", B, K, xdt)
    W = synth.normal((K, N), synth.seed_of(seed, K, N, "W"), 0.02, wdt)
    y, bm = sb.sfx_sparse_gemv(dev(x), dev(W), t=t, out_dtype=DT[out], flags=flags,
                               want_bitmap=True)
    m = O.magnitude_mask(to64(x), t)
    assert np.array_equal(bm.cpu().numpy(), pack_bitmap(m)), "fused mask differs"
    want = O.masked_gemv(to64(x), m, to64(W))
    if flags & sb.SFX_FLAG_GELU:
        want = O.gelu_erf(want)
    if flags & sb.SFX_FLAG_SWIGLU:
        want = O.silu(want[:, 0::2]) * want[:, 1::2]
        out = "f32"
    assert_close(to64(y), O.round_to(want, out), f"mma B={B} K={K} N={N} p={p}")
    return x, W, t, y


@pytest.mark.parametrize("B,K,N,p,wdt,xdt,out", [
    (2, 4096, 2048, 0.5, "bf16", "bf16", "bf16"),
    (3, 1000, 264, 0.3, "f16", "f16", "f32"),       # ragged K; N not a multiple of 64
    (4, 4096, 6144, 0.5, "bf16", "bf16", "bf16"),
    (5, 33, 136, 0.0, "bf16", "bf16", "f32"),       # tiny, dense: one partial K-block
    (8, 14336, 4096, 0.65, "bf16", "f32", "bf16"),  # fp32 inputs: hi + lo bf16 tiles
    (11, 3000, 1000, 0.5, "f16", "f32", "f16"),     # fp32 inputs with fp16 weights
    (16, 8192, 1024, 0.9, "bf16", "bf16", "bf16"),  # sparse union
    (16, 4096, 520, 0.0, "bf16", "bf16", "f32"),    # dense, N = 512 + 8
])
def test_union_mma_matches_oracle(B, K, N, p, wdt, xdt, out):
    case(B, K, N, p, wdt, xdt, out)


@pytest.mark.parametrize("chunks", [1, 2, 4, 8])
@pytest.mark.parametrize("B,K,N,p,wdt,xdt,out,flags", [
    (16, 4096, 1000, 0.5, "bf16", "bf16", "f32", 0),           # N % 64 != 0
    (5, 3000, 2056, 0.3, "f16", "f32", "f16", 0),              # fp32 x, ragged K
    (9, 2048, 4096, 0.4, "bf16", "bf16", "f32", sb.SFX_FLAG_SWIGLU),
])
def test_union_mma_every_tile_width(chunks, B, K, N, p, wdt, xdt, out, flags, monkeypatch):
    # 8 / chunks warps share each 64-column chunk and are summed in shared memory
    with sb.plan_overrides(mma_chunks=chunks):
        assert sb.sfx_gemv_plan(B, K, N, flags)["chunks"] == chunks
        case(B, K, N, p, wdt, xdt, out, flags=flags, seed=f"mma-c{chunks}")


def test_union_mma_epilogues():
    case(4, 2560, 1024, 0.4, "f16", "f16", "f32", flags=sb.SFX_FLAG_GELU, seed="mma-gelu")
    case(16, 4096, 28672, 0.5, "bf16", "bf16", "f32", flags=sb.SFX_FLAG_SWIGLU, seed="mma-gu")
    B, K, N = 6, 1024, 512
    x = synth.eval_draw("mma-umask", "x", B, K, "bf16")
    W = synth.normal((K, N), synth.seed_of("mma-umask", "W"), 0.02, "bf16")
    y = sb.sfx_sparse_gemv(dev(x), dev(W), t=1.1, flags=sb.SFX_FLAG_UNION_MASK,
                           out_dtype=torch.float32)
    u = O.union_mask(O.magnitude_mask(to64(x), 1.1))
    want = O.masked_gemv(to64(x), np.broadcast_to(u, (B, K)), to64(W))
    assert_close(to64(y), O.round_to(want, "f32"), "mma union-mask reading")


@pytest.mark.parametrize("B", [2, 16])
def test_union_mma_equals_cuda_core_path(B):
    K, N = 4096, 3072
    x = dev(synth.eval_draw("mma-vs-cc", "x", B, K, "bf16"))
    W = dev(synth.normal((K, N), synth.seed_of("mma-vs-cc", "W"), 0.02, "bf16"))
    y_mma = sb.sfx_sparse_gemv(x, W, t=0.9, out_dtype=torch.float32)
    y_cc = sb.sfx_sparse_gemv(x, W, t=0.9, out_dtype=torch.float32, flags=sb.SFX_FLAG_CUDA_CORES)
    assert_close(to64(y_mma), to64(y_cc), "mma vs CUDA cores")
    # the split sums are added in a fixed order: the same bits on every call
    assert torch.equal(y_mma, sb.sfx_sparse_gemv(x, W, t=0.9, out_dtype=torch.float32))


def test_union_mma_empty_union_gives_zero():
    B, K, N = 4, 2048, 1024
    x = synth.eval_draw("mma-empty", "x", B, K, "bf16")
    W = synth.normal((K, N), synth.seed_of("mma-empty", "W"), 0.02, "bf16")
    y = sb.sfx_sparse_gemv(dev(x), dev(W), t=float(x.abs().max()), out_dtype=torch.float32)
    assert torch.count_nonzero(y).item() == 0


@pytest.mark.parametrize("B", [3, 8, 16])
def test_ffn_swiglu_batched_on_mma(B):
    # both FFN stages (gate|up with the SwiGLU epilogue, then down on fp32 h)
    ffn_case(B, 1024, 3584, 0.5, seed=f"mma-ffn-b{B}")
