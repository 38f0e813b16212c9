"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds NO arithmetic of the method (no products, sums or
activations): it only draws seeded random numbers and rounds them to the
storage dtype.  Both the CUDA path's tests/benchmark and the CPU oracle's
tests draw their inputs from here, so the two sides see identical bits.

Recipe (one stream per operand, numpy PCG64, float32 draws, then one
round-to-nearest-even to the storage dtype):
  X  ~ N(0, 1)        seed + 0      [M, K]
  Wg ~ N(0, 1/K)      seed + 1      [N, K]   (std = 1/sqrt(K), applied in fp32)
  Wu ~ N(0, 1/K)      seed + 2      [N, K]
  dH ~ N(0, 1)        seed + 3      [n]
  G, U for the backward ~ N(0, 1)   seed + 4, seed + 5
The scale 1/K keeps G and U O(1), as nn.Linear-style initialisation does.
"""
from __future__ import annotations

import numpy as np
import torch

DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


def _draw(shape, seed: int, std: float = 1.0) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def normal(shape, seed: int, std: float = 1.0, dtype: str = "bf16") -> torch.Tensor:
    """CPU tensor of N(0, std^2) draws rounded (RNE) to `dtype`."""
    t = torch.from_numpy(_draw(tuple(shape), seed, std))
    return t.to(DTYPES[dtype]) if dtype != "f32" else t


def swiglu_inputs(M: int, K: int, N: int, dtype: str = "bf16", seed: int = 0):
    """(X [M,K], Wg [N,K], Wu [N,K]) on the CPU."""
    std_w = 1.0 / np.sqrt(K) if K > 0 else 1.0
    X = normal((M, K), seed + 0, 1.0, dtype)
    Wg = normal((N, K), seed + 1, std_w, dtype)
    Wu = normal((N, K), seed + 2, std_w, dtype)
    return X, Wg, Wu


def dswiglu_inputs(n: int, dtype: str = "bf16", seed: int = 0):
    """(dH, G, U), each [n] ~ N(0,1), on the CPU."""
    return (normal((n,), seed + 3, 1.0, dtype),
            normal((n,), seed + 4, 1.0, dtype),
            normal((n,), seed + 5, 1.0, dtype))


def integer_inputs(M: int, K: int, N: int, seed: int = 0, dtype: str = "bf16"):
    """Small-integer operands for bit-exact checks.

    X entries in {-1, 0, 1} except column 0, which is 16; Wg entries in
    {-1, 0, 1} except column 0, which is cw, the smallest power of two with
    16*cw >= K + 16, so every gate pre-activation is >= 17; Wu entries in
    {-2..2}.  Every operand is an integer exactly representable in bf16, and
    every product and partial sum is an integer below 2^24 for K <= 256, so
    any summation order gives the same fp32 result."""
    rng = np.random.Generator(np.random.PCG64(seed + 100))
    X = rng.integers(-1, 2, size=(M, K)).astype(np.float32)
    Wg = rng.integers(-1, 2, size=(N, K)).astype(np.float32)
    Wu = rng.integers(-2, 3, size=(N, K)).astype(np.float32)
    if K > 0:
        cw = 1
        while 16 * cw < K + 16:
            cw *= 2
        X[:, 0] = 16.0
        Wg[:, 0] = float(cw)
    conv = (lambda a: torch.from_numpy(a).to(DTYPES[dtype])) if dtype != "f32" \
        else torch.from_numpy
    return conv(X), conv(Wg), conv(Wu)


def ternary(shape, seed: int, density: float = 0.5, dtype: str = "bf16") -> torch.Tensor:
    """Entries in {-1, 0, +1}: nonzero with probability `density`, either
    sign equally likely.  For bit-exact checks of sums: every partial sum of
    such entries (and of their products) is a small integer, exact in fp32
    whatever the summation order."""
    rng = np.random.Generator(np.random.PCG64(seed + 200))
    mag = (rng.random(size=tuple(shape)) < density).astype(np.float32)
    sign = np.where(rng.random(size=tuple(shape)) < 0.5, -1.0, 1.0).astype(np.float32)
    t = torch.from_numpy(mag * sign)
    return t.to(DTYPES[dtype]) if dtype != "f32" else t
