"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module only draws random numbers and rounds them to bf16.  It holds none
of the method's arithmetic (no scales, no codes, no products), so it is the
one piece of code both sides may use.

Recipe (the decode workloads of the quantized linear layer):
  * activations X [M, K] ~ N(0, 1); optionally a fixed set of ceil(1% * K)
    distinct "outlier" input channels multiplied by 20 (chosen once per K and
    shared across M);
  * weights W [N, K] ~ N(0, 0.02);
  * drawn in fp32 with numpy's PCG64, then rounded to bf16 (round to nearest
    even).
Seeds: X uses the key (seed, M, K), W uses (seed + 1, N, K), the outlier
channel set (seed + 2, K).
"""
from __future__ import annotations

import math

import numpy as np
import torch

OUTLIER_FRACTION = 0.01
OUTLIER_GAIN = 20.0
WEIGHT_STD = 0.02


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def outlier_channels(K: int, seed: int) -> np.ndarray:
    n = int(math.ceil(OUTLIER_FRACTION * K))
    return np.sort(_rng(seed + 2, K).choice(K, size=n, replace=False))


def activations(M: int, K: int, seed: int, outliers: bool = True) -> torch.Tensor:
    """X [M, K] bf16 on the CPU."""
    x = _rng(seed, M, K).standard_normal((M, K), dtype=np.float32)
    if outliers:
        x[:, outlier_channels(K, seed)] *= np.float32(OUTLIER_GAIN)
    return _to_bf16(x)


def weights(N: int, K: int, seed: int, std: float = WEIGHT_STD) -> torch.Tensor:
    """W [N, K] bf16 on the CPU."""
    w = _rng(seed + 1, N, K).standard_normal((N, K), dtype=np.float32)
    w *= np.float32(std)
    return _to_bf16(w)


def uniform_bf16(shape, lo: float, hi: float, seed: int) -> torch.Tensor:
    """Uniform values rounded to bf16 (edge-case fixtures)."""
    a = _rng(seed, *shape).uniform(lo, hi, size=shape).astype(np.float32)
    return _to_bf16(a)
