"""The allocation-free GEMV entry point matches the oracle and the workspace one.

sfx_sparse_gemv_noalloc serves callers that cannot allocate device memory (a
plugin that is handed only inputs and outputs, or a framework that owns all
device memory); its scratch is a fixed device array inside the library. This
file is named so that pytest collects it last; it also passes on its own in a
fresh process.
"""
import ctypes
import math

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


def _call(x, W, t, y, flags=0, idx=None, cnt=None):
    # straight through the C ABI: only inputs, outputs and the stream
    B, K = x.shape
    N = W.shape[1]
    p = lambda v: None if v is None else ctypes.c_void_p(v.data_ptr())
    return sb.load().sfx_sparse_gemv_noalloc(
        p(x), sb._DT[x.dtype], B, K, p(W), sb._DT[W.dtype], N, float(t), p(idx), p(cnt), p(y),
        sb._DT[y.dtype], flags, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("B,K,N,t,dtype", [
    (1, 4096, 28672, 0.69, torch.bfloat16),   # gate|up-shaped, 50% sparse inputs
    (1, 14336, 4096, 0.36, torch.bfloat16),   # down-shaped
    (4, 2048, 4096, 0.69, torch.bfloat16),    # batch of 4, union of masks
    (1, 256, 512, 0.70, torch.float16),       # small fp16 GEMV
])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(B, K, N, t, dtype):
    sd = "f16" if dtype == torch.float16 else "bf16"
    W = synth.normal((K, N), synth.seed_of("noalloc", K, N), 0.02, sd, device="cuda")
    W64 = to64(W)
    ref_ws = sb.Workspace()
    for call in range(2):  # two calls in a row: the shared array must not leak state
        x = synth.eval_draw("noalloc", f"{K}", B, K, sd, draw=64 + 7 * call)
        want = O.masked_gemv(to64(x), O.magnitude_mask(to64(x), t), W64)
        same = sb.sfx_sparse_gemv(x.cuda(), W, t=t, out_dtype=torch.float32, ws=ref_ws)
        y = torch.full((B, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(x.cuda(), W, t, y) == 0
        torch.cuda.synchronize()
        assert_close(to64(y), O.round_to(want, "f32"), f"call {call} vs oracle")
        assert_close(to64(y), to64(same), f"call {call} vs workspace entry point")
    assert ref_ws.status() == 0


def test_noalloc_shape_sequence_leaves_no_stale_counters():
    # a wide batch-union call (many column tiles), a narrow one, then the wide
    # one again: counters left by one shape must not pick the wrong last CTA
    # of another
    seq = [(4, 2048, 28672), (1, 1024, 512), (4, 2048, 28672), (2, 4096, 2048)]
    t = 0.69
    for i, (B, K, N) in enumerate(seq):
        W = synth.normal((K, N), synth.seed_of("noalloc-seq", K, N), 0.02, "bf16", device="cuda")
        x = synth.eval_draw("noalloc-seq", f"{K}", B, K, "bf16", draw=64 + i)
        y = torch.full((B, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(x.cuda(), W, t, y) == 0
        torch.cuda.synchronize()
        want = O.masked_gemv(to64(x), O.magnitude_mask(to64(x), t), to64(W))
        assert_close(to64(y), O.round_to(want, "f32"), f"call {i} {B}x{K}x{N}")


def test_noalloc_index_list_mode_twice():
    K, N = 10240, 2560
    W = synth.normal((K, N), synth.seed_of("noalloc-idx"), 0.02, "f16", device="cuda")
    h = synth.normal((K,), synth.seed_of("noalloc-idx", "h"), 1.0, "f32")
    for k in (3072, 7168):
        idx = torch.arange(0, K, K // k, dtype=torch.int32)[:k].contiguous()
        cnt = torch.tensor([idx.numel()], dtype=torch.int32, device="cuda")
        m = np.zeros(K, bool)
        m[idx.numpy()] = True
        want = O.masked_gemv(to64(h)[None], m[None], to64(W))[0]
        y = torch.empty((1, N), dtype=torch.float32, device="cuda")
        assert _call(h.cuda()[None], W, -math.inf, y, idx=idx.cuda(), cnt=cnt) == 0
        torch.cuda.synchronize()
        assert_close(to64(y[0]), O.round_to(want, "f32"), f"k={k}")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # B = 16 over 57344 columns needs tens of MB of partial sums: more than
    # the fixed array holds, so the call is refused before any launch.
    x = torch.zeros((16, 1024), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((1024, 57344), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((16, 57344), dtype=torch.bfloat16, device="cuda")
    assert _call(x, W, 0.5, y) == -7
    assert torch.count_nonzero(y).item() == 0
