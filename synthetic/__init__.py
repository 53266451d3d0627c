"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and the bench.

This module draws random numbers and rounds them to storage precisions. It holds
none of the transform's or the layer's arithmetic, so importing it from both the
oracle side and the CUDA side keeps the two independent.

Recipe (the workloads of "Memory-Efficient Training with In-Place FFT
Implementation"; the pages give shapes only):
  * every value is drawn as float64 from numpy's PCG64 generator seeded with an
    integer, i.i.d. N(0, sigma^2);
  * fp32 inputs are that float64 rounded once to float32 (round to nearest even);
  * bf16 inputs are that float64 rounded once to bfloat16 (round to nearest even),
    carried as raw uint16 bit patterns so that the GPU and the oracle see the same
    bits; the oracle reads the exact float64 value of those bits.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "normal",
    "round_to_f32",
    "round_to_bf16",
    "bf16_bits_to_f64",
    "Sample",
    "sample",
]


def normal(seed: int, shape, sigma: float = 1.0) -> np.ndarray:
    """float64 i.i.d. N(0, sigma^2) of `shape` from PCG64(seed)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal(size=shape, dtype=np.float64) * sigma


def round_to_f32(v: np.ndarray) -> np.ndarray:
    """Round float64 to float32 (nearest even); returns float32."""
    return np.asarray(v, dtype=np.float64).astype(np.float32)


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 to bfloat16 (nearest, ties to even) in one step.

    Returns the uint16 bit patterns. The rounding is done on the float64 value
    directly (8 significant bits), not via float32, so there is no double rounding.
    Values beyond the bf16 range saturate to +-inf; values below the smallest
    normal are flushed to signed zero (N(0,1) data never reaches either).
    """
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                      # v = m * 2**e, 0.5 <= |m| < 1
    q = np.rint(np.ldexp(m, 8))             # 8 significant bits, ties to even
    r = np.ldexp(q, e - 8)                  # exact in float64
    tiny = np.abs(r) < np.ldexp(1.0, -126)
    r = np.where(tiny, np.copysign(0.0, v), r)
    big = np.abs(r) >= np.ldexp(1.0, 128)
    r = np.where(big, np.copysign(np.inf, v), r)
    bits32 = r.astype(np.float32).view(np.uint32)   # exact: r is a bf16 value
    return (bits32 >> 16).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact float64 value of bfloat16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


class Sample:
    """One seeded tensor in a storage dtype plus its exact float64 value.

    `stored` is float32 (dtype 'f32') or uint16 bf16 bits (dtype 'bf16');
    `exact` is the float64 value the stored data represents.
    """

    def __init__(self, stored: np.ndarray, exact: np.ndarray, dtype: str):
        self.stored = stored
        self.exact = exact
        self.dtype = dtype


def sample(seed: int, shape, dtype: str, sigma: float = 1.0) -> Sample:
    """Draw N(0, sigma^2) in float64 and round it once to `dtype` ('f32' or 'bf16')."""
    v = normal(seed, shape, sigma)
    if dtype == "f32":
        s = round_to_f32(v)
        return Sample(s, s.astype(np.float64), dtype)
    if dtype == "bf16":
        s = round_to_bf16(v)
        return Sample(s, bf16_bits_to_f64(s), dtype)
    raise ValueError(f"unknown dtype {dtype!r}")
