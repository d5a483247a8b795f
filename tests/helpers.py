"""Shared test utilities: tolerance checks, mask packing, GPU gating."""
import numpy as np
import pytest
import torch

# Floating-point bar for outputs (fp32 accumulation vs the fp64 oracle rounded
# to the output dtype): relative L2 error <= 1e-3 and max-abs error <= 1e-2 max|y|.
REL_L2 = 1e-3
MAX_ABS_FRAC = 1e-2


def has_gpu():
    return torch.cuda.is_available()


def to64(t) -> np.ndarray:
    """Exact float64 values of a tensor (any float dtype), on the host."""
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(got, want, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    err = got - want
    nrm = np.linalg.norm(want)
    rel = np.linalg.norm(err) / nrm if nrm > 0 else np.linalg.norm(err)
    scale = np.abs(want).max() if want.size else 0.0
    mx = np.abs(err).max() if err.size else 0.0
    assert rel <= REL_L2, f"{what}: rel L2 {rel:.3e} > {REL_L2}"
    assert mx <= MAX_ABS_FRAC * max(scale, 1e-30) or (scale == 0 and mx == 0), \
        f"{what}: max abs {mx:.3e} > {MAX_ABS_FRAC} * {scale:.3e}"
    return rel, mx


def pack_bitmap(mask: np.ndarray) -> np.ndarray:
    """bool [B x K] -> int32 [B x ceil(K/32)], bit (i % 32) of word i // 32."""
    mask = np.atleast_2d(np.asarray(mask, dtype=bool))
    B, K = mask.shape
    W = (K + 31) // 32
    padded = np.zeros((B, W * 32), dtype=np.uint64)
    padded[:, :K] = mask
    words = (padded.reshape(B, W, 32) << np.arange(32, dtype=np.uint64)).sum(axis=2)
    return words.astype(np.uint32).view(np.int32)


gpu = pytest.mark.gpu
