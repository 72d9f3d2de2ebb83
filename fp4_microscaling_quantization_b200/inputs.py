"""Seeded synthetic input tensors (bf16 bit patterns) for tests and the benchmark.

This module only draws random numbers and rounds them to bf16; it holds none of
the quantization arithmetic.  The same bytes are fed to the CUDA library and to
the CPU oracle.

Distributions follow the workloads the pages describe: heavy-tailed activations
with sparse large outliers and near-Laplacian weights ("Portable FP4
quantization", §3.1 Table 4), shaped like Llama-8B / 70B projections.

Recipe (also stated in the design notes):
  * ``numpy.random.default_rng(seed)``; tensors are drawn in row-major order in
    chunks of rows, A before W;
  * Laplace(0, b) = b * (E1 - E2), E1, E2 ~ Exp(1) drawn as float32;
  * Student-t(nu) from ``standard_t`` (float64) cast to float32;
  * "p outliers x f": a Bernoulli(p) mask from the same generator, masked
    entries multiplied by f;
  * "c outlier channels x f": round(c * cols) distinct columns (drawn without
    replacement) multiplied by f in every row;
  * float32 -> bf16 by round-to-nearest-even on the bit pattern.
"""
from __future__ import annotations

import numpy as np

_CHUNK = 1 << 22  # elements per draw, bounds host memory for large tensors


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even), returned as uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _laplace(rng, n, scale):
    e1 = rng.standard_exponential(n, dtype=np.float32)
    e2 = rng.standard_exponential(n, dtype=np.float32)
    return (e1 - e2) * np.float32(scale)


def _student_t(rng, n, nu):
    return rng.standard_t(nu, n).astype(np.float32)


def draw(rng, rows: int, cols: int, dist: str, scale: float = 1.0, nu: float = 3.0,
         outlier_p: float = 0.0, outlier_mult: float = 1.0,
         channel_frac: float = 0.0, channel_mult: float = 1.0) -> np.ndarray:
    """One (rows, cols) bf16 tensor (uint16 bit patterns)."""
    out = np.empty((rows, cols), np.uint16)
    flat = out.reshape(-1)
    n = rows * cols
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        if dist == "laplace":
            v = _laplace(rng, m, scale)
        elif dist == "student_t":
            v = _student_t(rng, m, nu) * np.float32(scale)
        else:
            raise ValueError(dist)
        if outlier_p > 0.0:
            mask = rng.random(m, dtype=np.float32) < np.float32(outlier_p)
            v[mask] *= np.float32(outlier_mult)
        flat[s:s + m] = f32_to_bf16_bits(v)
    if channel_frac > 0.0:
        nch = int(round(channel_frac * cols))
        ch = np.sort(rng.choice(cols, size=nch, replace=False))
        v = bf16_bits_to_f32(out[:, ch]) * np.float32(channel_mult)
        out[:, ch] = f32_to_bf16_bits(v)
    return out


# ---- the workloads --------------------------------------------------------------
def tiny_linear(seed: int = 0):
    """MXFP4 W4A4 linear, tiny: A 128x512 Laplace(0,1) with 1% outliers x20,
    W 256x512 Laplace(0,0.02)."""
    rng = np.random.default_rng(seed)
    a = draw(rng, 128, 512, "laplace", 1.0, outlier_p=0.01, outlier_mult=20.0)
    w = draw(rng, 256, 512, "laplace", 0.02)
    return a, w


def quant_sweep(rows: int = 1024, cols: int = 131072, seed: int = 2):
    """Heavy-tailed tensor: Student-t(3) with 1% outliers x20."""
    rng = np.random.default_rng(seed)
    return draw(rng, rows, cols, "student_t", 1.0, nu=3.0, outlier_p=0.01, outlier_mult=20.0)


def rotate_acts(rows: int = 8192, cols: int = 4096, seed: int = 3):
    """Laplace(0,1) activations with 1% outlier channels x50."""
    rng = np.random.default_rng(seed)
    return draw(rng, rows, cols, "laplace", 1.0, channel_frac=0.01, channel_mult=50.0)


def decode_linear(m: int, n: int, k: int, seed: int = 4):
    """Decode shape: A m x k Laplace(0,1), W n x k Laplace(0,0.02)."""
    rng = np.random.default_rng(seed)
    a = draw(rng, m, k, "laplace", 1.0)
    w = draw(rng, n, k, "laplace", 0.02)
    return a, w


def prefill_linear(m: int = 8192, n: int = 28672, k: int = 8192, seed: int = 5):
    """Prefill shape: A m x k Laplace(0,1) with 1% outliers x20, W n x k
    Laplace(0,0.02)."""
    rng = np.random.default_rng(seed)
    a = draw(rng, m, k, "laplace", 1.0, outlier_p=0.01, outlier_mult=20.0)
    w = draw(rng, n, k, "laplace", 0.02)
    return a, w


def table5_activation(n: int = 131072, outlier_p: float = 0.01, seed: int = 11):
    """'Portable FP4 quantization' Table 4 activation tensor: 0.42 * t(5)
    body plus N(0, 6^2) added at a Bernoulli(outlier_p) subset (fp32)."""
    rng = np.random.default_rng(seed)
    x = 0.42 * rng.standard_t(5, n)
    mask = rng.random(n) < outlier_p
    x[mask] += rng.normal(0.0, 6.0, int(mask.sum()))
    return x.astype(np.float32)


def table5_weight(n: int = 131072, outlier_p: float = 0.003, seed: int = 12):
    """Table 4 weight tensor: N(0, 0.55^2) body plus N(0, 6^2) outliers."""
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 0.55, n)
    mask = rng.random(n) < outlier_p
    x[mask] += rng.normal(0.0, 6.0, int(mask.sum()))
    return x.astype(np.float32)
