"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark's CPU baseline.

This module draws random numbers and formats them; it holds none of the
BitLinear arithmetic (no scale, no rounding to integers, no contraction).
Both the CUDA path and the CPU oracle receive exactly the arrays made here.

Distributions follow the shapes of BitNet b1.58 2B4T layers (BitNetConfig on
the BitNet model page: hidden 2560, intermediate 6912, initializer_range 0.02):

* latent weights: N(0, sigma), sigma = 0.02, fp32;
* activations: N(0, 1) rounded to bf16 (round-half-to-even on the fp32 bits);
  optional variants:
  - ``outliers``: 4 channel indices drawn once per seed (without replacement)
    are multiplied by 20 in every token;
  - ``student_t_rows``: every 8th row (m % 8 == 7) is Student-t with 3 degrees
    of freedom instead of normal (heavy-tailed tokens).

The generator is numpy's PCG64 seeded with the integer seed given.
"""
import numpy as np

SIGMA_W = 0.02
OUTLIER_CHANNELS = 4
OUTLIER_SCALE = 20.0


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def latent_weights(n: int, k: int, seed: int, sigma: float = SIGMA_W) -> np.ndarray:
    """fp32 [n][k] ~ N(0, sigma)."""
    return (rng(seed).standard_normal((n, k), dtype=np.float64) * sigma).astype(np.float32)


def activations(m: int, k: int, seed: int, kind: str = "normal") -> np.ndarray:
    """bf16 bit patterns (uint16) [m][k]."""
    g = rng(seed)
    x = g.standard_normal((m, k), dtype=np.float64)
    if kind == "normal":
        pass
    elif kind == "outliers":
        ch = g.choice(k, size=min(OUTLIER_CHANNELS, k), replace=False)
        x[:, ch] *= OUTLIER_SCALE
    elif kind == "student_t_rows":
        rows = np.arange(m) % 8 == 7
        if rows.any():
            x[rows] = g.standard_t(3, size=(int(rows.sum()), k))
    else:
        raise ValueError(f"unknown activation kind {kind!r}")
    return f32_to_bf16_bits(x.astype(np.float32))


def activations_f32(m: int, k: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """fp32 [m][k] ~ N(0, scale) (for inputs that arrive in fp32, e.g. a gated FFN output)."""
    return (rng(seed).standard_normal((m, k), dtype=np.float64) * scale).astype(np.float32)
