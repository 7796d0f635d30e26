"""Seeded synthetic inputs for the W4A4 quantized-linear workloads.

This module is shared by the tests, the oracle-side checks and the benchmark.  It
holds random draws and bit-level dtype plumbing only: no quantization rule, no
codec, no GEMM.  Everything the method computes from these draws lives twice,
once in ``oracle/`` (CPU, fp64) and once in the CUDA library, and never here.

Generators follow published methods: numpy's PCG64 bit generator
(``numpy.random.default_rng``), its Fisher-Yates ``permutation``, its normal
sampler and its Student-t sampler.  bf16 rounding of the draws uses torch's CPU
round-to-nearest-even conversion.
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "rng", "to_bf16_bits", "bf16_bits_to_f64", "f32_to_bf16_bits", "pick_channels",
    "activations_bf16", "student_t", "uniform_nibble_bytes", "uniform_bytes",
]


def rng(seed: int) -> np.random.Generator:
    """PCG64 generator for one workload seed."""
    return np.random.default_rng(int(seed))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round a float array to bf16 (RNE, via torch) and return the raw uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    return to_bf16_bits(a)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def pick_channels(g: np.random.Generator, K: int, frac: float) -> np.ndarray:
    """round(frac*K) distinct channels by a seeded Fisher-Yates shuffle, ascending."""
    count = int(round(frac * K))
    return np.sort(g.permutation(K)[:count])


def activations_bf16(seed: int, M: int, K: int, outlier_frac: float, outlier_scale: float,
                     channels_seed: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """X ~ N(0,1) [M,K] with a seeded set of outlier channels scaled by ``outlier_scale``.

    The outlier channels depend on ``channels_seed`` (default: ``seed``) only, so every M of
    one workload shares the same channels.  Returns (bf16 bits [M,K], channel indices).
    """
    cs = seed if channels_seed is None else channels_seed
    ch = pick_channels(rng(cs * 7919 + 1), K, outlier_frac)
    x = rng(seed * 1_000_003 + M).standard_normal((M, K))
    x[:, ch] *= outlier_scale
    return to_bf16_bits(x), ch


def student_t(seed: int, shape: tuple[int, ...], nu: float) -> np.ndarray:
    """Student-t(nu) draws in float64."""
    return rng(seed).standard_t(nu, size=shape)


def uniform_nibble_bytes(seed: int, rows: int, nibbles: int) -> np.ndarray:
    """Uniform random 4-bit codes (all 16 values), packed two per byte: [rows, nibbles/2] uint8."""
    assert nibbles % 2 == 0
    return rng(seed).integers(0, 256, size=(rows, nibbles // 2), dtype=np.uint8)


def uniform_bytes(seed: int, shape: tuple[int, ...], lo: int, hi: int) -> np.ndarray:
    """Uniform random bytes in the inclusive range [lo, hi]."""
    return rng(seed).integers(lo, hi + 1, size=shape, dtype=np.uint8)
