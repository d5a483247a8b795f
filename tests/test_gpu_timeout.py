"""Bounded waits run out without harming the GPU context (GPU).

Kernels that hand data between warps through mbarriers give up on a wait
after a limit, raise SFX_DEV_TIMEOUT in the workspace status word, wait (at
most 20 ms) for the copies and MMAs they started, free their tensor memory and
return. Here the test hook SFX_PLAN_TEST_STALL leaves the first stage of the
dense kernel's ring without its second producer's arrival -- a barrier that
nothing completes -- and the wait limit is 2 ms; the test reads the status
word, then turns the hook off, restores the limit, re-initialises the
workspace and checks that the same call matches the fp64 oracle: the context
is still usable.
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
    yield
    sb.sfx_set_wait_limit_ns(0)


@pytest.mark.parametrize("mode", [sb.DENSE_ONLY, sb.DENSE_ONLY_TCGEN05])
def test_wait_limit_runs_out_and_the_context_survives(mode):
    B, K, N, t = 16, 2048, 4096, 0.5
    x = synth.eval_draw("timeout", "x", B, K, "bf16")
    W = synth.normal((K, N), synth.seed_of("timeout", "W"), 0.02, "bf16")
    xd, Wd = x.cuda(), W.cuda()
    ws = sb.Workspace()
    ws.reserve(sb.sfx_workspace_bytes(sb.SFX_OP_SPARSE_GEMV, B, K, N, sb.SFX_BF16))
    with sb.plan_overrides(dense=mode):
        sb.sfx_set_wait_limit_ns(2_000_000)
        try:
            with sb.plan_overrides(test_stall=1):
                sb.sfx_sparse_gemv(xd, Wd, t=t, out_dtype=torch.float32, ws=ws)
            bits = ws.status()  # synchronises, reads and clears the status word
        finally:
            sb.sfx_set_wait_limit_ns(0)
        assert bits & sb.SFX_DEV_TIMEOUT, bits
        # the counters may be mid-count after a timeout: re-initialise, run again
        assert sb.load().sfx_workspace_init(ctypes.c_void_p(ws.buf.data_ptr()), ws.buf.numel(),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
        y = sb.sfx_sparse_gemv(xd, Wd, t=t, out_dtype=torch.float32, ws=ws)
        assert ws.status() == 0
    want = O.masked_gemv(to64(x), O.magnitude_mask(to64(x), t), to64(W))
    assert_close(to64(y), O.round_to(want, "f32"), "after the timeout")
