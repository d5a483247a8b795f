"""Block error curves for the greedy allocation, against the oracle (GPU).

"TEAL: Training-Free Activation Sparsity in Large Language Models", slide 10:
the greedy allocation needs each block's l2 activation error at each sparsity
level. sfx_block_error_curve computes it on the GPU (exact calibration, the
sparse GEMV, an fp64 sum of squared changes); the thresholds must equal the
oracle's bit for bit. The errors are differences of two fp32 products of up to
K = 2048 terms, each off by about sqrt(K) 2^-24 of the output norm, so they
agree within 1e-4 relative plus 1e-5 of the dense output's norm. The
allocation built from the GPU's curves by sfx_greedy_allocate must equal the
oracle's allocation from its own curves.
"""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import to64
from sparse_input_gemv_b200 import binding as sb
from sparse_input_gemv_b200 import synth

pytestmark = pytest.mark.gpu

LEVELS = [round(0.05 * i, 2) for i in range(20)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sb.load()


def curve_case(name, K, N, xdt, wdt="bf16", scale=1.0):
    X = synth.calib_draws("alloc", name, 64, K, xdt) if scale == 1.0 else \
        synth.to_storage(synth.calib_draws("alloc", name, 64, K, "f32").double() * scale, xdt)
    W = synth.normal((K, N), synth.seed_of("alloc", name, "W"), 0.02, wdt)
    err, thr = sb.sfx_block_error_curve(X.cuda(), W.cuda(), LEVELS)
    want_err, want_thr = O.block_error_curve(to64(X), to64(W), LEVELS)
    assert [float(np.float32(t)) for t in want_thr] == thr
    assert err[0] == 0.0
    dense = np.linalg.norm(to64(X) @ to64(W))
    np.testing.assert_allclose(err, want_err, rtol=1e-4, atol=1e-5 * dense)
    return err, want_err


@pytest.mark.parametrize("name,K,N,xdt", [("qkv", 1024, 1536, "bf16"), ("down", 2048, 512, "f32"),
                                          ("ragged", 1000, 264, "bf16")])
def test_error_curve_matches_oracle(name, K, N, xdt):
    curve_case(name, K, N, xdt)


def test_allocation_from_gpu_curves_equals_oracle_allocation():
    # three sites with different weights and input scales, target 50 %
    sites = [("s0", 1024, 2048, 1.0), ("s1", 1024, 512, 3.0), ("s2", 2048, 1024, 0.5)]
    got_curves, want_curves, weights = [], [], []
    for name, K, N, scale in sites:
        g, w = curve_case(name, K, N, "bf16", scale=scale)
        got_curves.append(g)
        want_curves.append(w)
        weights.append(K * N)
    step = 0.05
    got = sb.sfx_greedy_allocate(got_curves, weights, step, 0.5)
    want = O.greedy_allocate(np.array(want_curves), np.array(weights, float), step, 0.5)
    assert got == want.tolist(), (got, want)
    assert O.overall_sparsity(np.array(got) * step, weights) >= 0.5 - 1e-12
