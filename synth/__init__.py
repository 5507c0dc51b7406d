"""Seeded synthetic inputs for the FusedBitLinear projection.

This module draws random numbers and describes workload shapes; it holds none of the
projection's arithmetic.  It is the one module that both the oracle side (tests) and the
CUDA side (tests, bench) use, so both always see the same bits.

Generator: numpy's Philox counter-based bit generator, keyed by an integer seed and a
stream label, so every tensor of a workload has its own reproducible stream.
"""
import zlib

import numpy as np

from .workloads import WORKLOADS, Projection, Workload  # noqa: F401


def _rng(seed: int, label: str) -> np.random.Generator:
    key = zlib.crc32(label.encode()) & 0xFFFFFFFF
    return np.random.Generator(np.random.Philox(key=[int(seed) & 0xFFFFFFFFFFFFFFFF, key]))


def normal(seed: int, label: str, shape, std: float = 1.0, dtype=np.float16) -> np.ndarray:
    """N(0, std^2) samples drawn in float64, then rounded to ``dtype``."""
    r = _rng(seed, label)
    a = r.standard_normal(size=shape, dtype=np.float64)
    if std != 1.0:
        a *= std
    return a.astype(dtype)


def activations(seed: int, label: str, T: int, K: int, dtype=np.float16,
                outlier_frac: float = 0.0, outlier_scale: float = 20.0) -> np.ndarray:
    """x ~ N(0,1) [T,K]; optionally a Bernoulli(outlier_frac) mask of entries scaled by
    ``outlier_scale`` (the prefill workload's outliers)."""
    r = _rng(seed, "x/" + label)
    a = r.standard_normal(size=(T, K), dtype=np.float64)
    if outlier_frac > 0.0:
        m = r.random(size=(T, K)) < outlier_frac
        a[m] *= outlier_scale
    return a.astype(dtype)


def weights(seed: int, label: str, N: int, K: int, std: float = 0.02,
            dtype=np.float32) -> np.ndarray:
    """Full-precision latent weights W ~ N(0, std^2) [N,K] (out_features x in_features)."""
    return normal(seed, "w/" + label, (N, K), std=std, dtype=dtype)


def norm_weight(seed: int, label: str, K: int, ones: bool = True) -> np.ndarray:
    """RMSNorm weight g [K]: all ones (every workload), or U(0.5, 1.5) for the tests that
    exercise a non-trivial g."""
    if ones:
        return np.ones(K, dtype=np.float32)
    r = _rng(seed, "g/" + label)
    return (0.5 + r.random(K)).astype(np.float32)


def int8_codes(seed: int, label: str, T: int, K: int) -> np.ndarray:
    """Uniform int8 codes in [-127, 127] (for the accumulator-only checks)."""
    r = _rng(seed, "q/" + label)
    return r.integers(-127, 128, size=(T, K), dtype=np.int16).astype(np.int8)


def ternary(seed: int, label: str, N: int, K: int, p_zero: float = 1.0 / 3) -> np.ndarray:
    """Ternary codes in {-1,0,1} with P(0) = p_zero."""
    r = _rng(seed, "c/" + label)
    u = r.random(size=(N, K))
    c = np.where(u < p_zero, 0, np.where(u < (1 + p_zero) / 2, -1, 1))
    return c.astype(np.int8)
