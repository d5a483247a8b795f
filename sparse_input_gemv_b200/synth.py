"""Seeded synthetic inputs for the activation-sparse GEMV / FFN path.

This module only draws random numbers and rounds them to a storage dtype. It
holds none of the method's arithmetic (no masking, selection or products), so
it is the one module that both the CUDA path's tests/bench and the CPU oracle
use to obtain the *same* input bits.

Distributions follow the workloads the source pages describe:

* activations x ~ Laplace(0, 1) -- the heavy-tailed block inputs that TEAL
  ("TEAL: Training-Free Activation Sparsity in Large Language Models",
  slide 7 "activation distribution analysis") reports for MLP and attention
  inputs; drawn by the inverse CDF of a uniform;
* weights W ~ N(0, 0.02^2);
* attribution gradients g ~ N(0, 1), GLASS score vectors |N(0, 1)|, MoE
  router logits ~ N(0, 1);
* a correlated-token variant of x for batched decoding: x_bi = s_i z_bi with
  z_bi ~ Laplace(0, 1) per token and a per-neuron scale s_i = exp(1.5 n_i),
  n_i ~ N(0, 1), shared by the tokens. The pages give no overlap between the
  masks of different tokens; the spread 1.5 makes that overlap (pairwise
  Jaccard 0.56 at half sparsity) fall in the 0.52-0.60 range that GLASS
  ("GLASS: Global-Local Aggregation for inference-time Sparsification",
  oracle-overlap analysis) reports between its masks and the oracle set.

Seeds are derived from a string key (workload, tensor name, draw number) by a
stable hash, so a tensor is reproducible from its name alone. CPU draws use
numpy's counter-based Philox generator. Very large weights can be drawn on a
CUDA device with torch's Philox generator instead (``device="cuda"``); those
values differ from the CPU draw of the same key but are just as reproducible,
and a test then copies the device tensor back to feed the oracle.
"""
from __future__ import annotations

import hashlib
import numpy as np
import torch

__all__ = [
    "seed_of", "laplace", "normal", "abs_normal", "to_storage",
    "STORAGE_DTYPES", "calib_draws", "eval_draw", "CORR_SIGMA", "correlated_draws",
]

STORAGE_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def seed_of(*parts) -> int:
    """Stable 63-bit seed from a tuple of names/numbers (blake2b of 'a|b|c')."""
    key = "|".join(str(p) for p in parts).encode()
    return int.from_bytes(hashlib.blake2b(key, digest_size=8).digest(), "little") >> 1


def _np_gen(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=seed))


def _torch_gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def to_storage(a, dtype: str) -> torch.Tensor:
    """Round an fp32/fp64 array to the storage dtype (round-to-nearest-even)."""
    t = a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a))
    return t.to(STORAGE_DTYPES[dtype]).contiguous()


def _uniform_open(shape, seed, device):
    """Uniform draws in the open interval (0, 1)."""
    if device == "cpu":
        u = _np_gen(seed).random(size=shape, dtype=np.float64)
        u = np.clip(u, 1e-300, None)
        return torch.from_numpy(u)
    u = torch.rand(shape, generator=_torch_gen(seed, device), device=device,
                   dtype=torch.float64)
    return u.clamp_min(1e-300)


def laplace(shape, seed: int, dtype: str = "bf16", scale: float = 1.0,
            device: str = "cpu") -> torch.Tensor:
    """Laplace(0, scale) by inverse CDF of u ~ U(0,1), rounded to `dtype`."""
    u = _uniform_open(shape, seed, device) - 0.5
    x = -scale * torch.sign(u) * torch.log1p(-2.0 * u.abs())
    return to_storage(x, dtype)


def normal(shape, seed: int, std: float = 1.0, dtype: str = "bf16",
           device: str = "cpu") -> torch.Tensor:
    """N(0, std^2) rounded to `dtype`."""
    if device == "cpu":
        x = torch.from_numpy(_np_gen(seed).standard_normal(size=shape) * std)
    else:
        x = torch.randn(shape, generator=_torch_gen(seed, device), device=device,
                        dtype=torch.float32) * std
    return to_storage(x, dtype)


def abs_normal(shape, seed: int, dtype: str = "f32", device: str = "cpu") -> torch.Tensor:
    """|N(0, 1)| rounded to `dtype` (stand-in importance / score vectors)."""
    return normal(shape, seed, 1.0, dtype, device).abs()


def calib_draws(workload: str, site: str, S: int, K: int, dtype: str,
                device: str = "cpu") -> torch.Tensor:
    """S calibration draws [S x K] of a site's input activations (draws 0..S-1)."""
    rows = [laplace((K,), seed_of(workload, site, "draw", s), dtype, device=device)
            for s in range(S)]
    return torch.stack(rows)


def eval_draw(workload: str, site: str, B: int, K: int, dtype: str, draw: int = 64,
              device: str = "cpu") -> torch.Tensor:
    """Evaluation activations [B x K]; draws start at 64, after the calibration set."""
    rows = [laplace((K,), seed_of(workload, site, "draw", draw + b), dtype, device=device)
            for b in range(B)]
    return torch.stack(rows)


CORR_SIGMA = 1.5  # log-normal spread of the shared per-neuron scales


def correlated_draws(workload: str, site: str, B: int, K: int, dtype: str, draw: int = 64,
                     sigma: float = CORR_SIGMA) -> torch.Tensor:
    """Tokens [B x K] sharing per-neuron scales: x_bi = exp(sigma n_i) z_bi.

    n ~ N(0, 1) is drawn once per (workload, site); z_b ~ Laplace(0, 1) per
    token from the same draw numbers as eval_draw (draws 0..63 calibrate).
    """
    n = _np_gen(seed_of(workload, site, "neuron-scales")).standard_normal(size=(K,))
    scale = torch.from_numpy(np.exp(sigma * n))
    rows = []
    for b in range(B):
        u = _uniform_open((K,), seed_of(workload, site, "draw", draw + b), "cpu") - 0.5
        z = -torch.sign(u) * torch.log1p(-2.0 * u.abs())
        rows.append(to_storage(scale * z, dtype))
    return torch.stack(rows)
