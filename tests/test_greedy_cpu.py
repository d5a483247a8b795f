"""sfx_greedy_allocate (host logic, no GPU) against the oracle's greedy rounds.

"TEAL: Training-Free Activation Sparsity in Large Language Models", slide 10:
every block starts dense and each round raises the block whose l2 error grows
least (per unit of model-wide sparsity bought) until the model-wide sparsity
reaches the target. The library's host
routine and the oracle are separate implementations; on the same error curves
they must pick the same level for every block.
"""
import numpy as np
import pytest

import oracle as O
from sparse_input_gemv_b200 import binding as sb


@pytest.fixture(scope="module", autouse=True)
def _lib():
    sb.load()


@pytest.mark.parametrize("seed", range(12))
def test_greedy_matches_oracle_on_random_curves(seed):
    rng = np.random.default_rng(seed)
    M, P = int(rng.integers(1, 7)), int(rng.integers(2, 21))
    step = 1.0 / (P - 1) if seed % 2 else 0.05
    if seed % 3 == 0:   # growing increments (convex)
        inc = np.sort(rng.uniform(0, 2, size=(M, P - 1)), axis=1)
    else:               # arbitrary non-negative increments
        inc = rng.uniform(0, 2, size=(M, P - 1))
    err = np.concatenate([np.zeros((M, 1)), np.cumsum(inc, axis=1)], axis=1)
    weights = rng.uniform(0.5, 4.0, size=M) if seed % 4 else np.ones(M)
    for target in (0.0, 0.1, 0.33, 0.5, 0.75, 0.9, 1.5):
        got = sb.sfx_greedy_allocate(err.tolist(), weights.tolist(), step, target)
        want = O.greedy_allocate(err, weights, step, target)
        assert got == want.tolist(), (seed, target, got, want)


def test_greedy_ties_go_to_the_lower_block():
    err = [[0.0, 1.0, 2.0], [0.0, 1.0, 2.0]]
    assert sb.sfx_greedy_allocate(err, [1, 1], 0.5, 0.25) == [1, 0]


def test_greedy_rejects_bad_arguments():
    with pytest.raises(sb.SfxError):
        sb.sfx_greedy_allocate([[0.0, 1.0]], [0.0], 0.5, 0.5)    # weights sum to 0
    with pytest.raises(sb.SfxError):
        sb.sfx_greedy_allocate([[0.0, 1.0]], [1.0], 0.0, 0.5)    # step must be > 0
