"""W4A4 GEMM reference (oracle; test infrastructure only).

y[m, n] = sum_k deq(x)[m, k] * deq(w)[n, k] in float64, the plain definition of the quantized
linear layer y = X W^T that all five pages share (PRQuant, §4 "Kernel design for efficient
inference": one MXFP4 GEMM over the quantized operands; MXCode abstract: MX-native W4A4
operands).  The dequantized operands are exact in float64, each product is exact, and the
float64 sum is within K * 2^-53 relative of the exact sum, far inside the float tolerance.

The tolerance scale t[m, n] = sum_k |deq x[m,k] * deq w[n,k]| bounds an fp32-accumulated
result: |y_gpu - y| <= 1e-5 * t per element before the bf16 cast.
"""
from __future__ import annotations

import numpy as np


def gemm_ref(xdeq: np.ndarray, wdeq: np.ndarray) -> np.ndarray:
    return np.asarray(xdeq, np.float64) @ np.asarray(wdeq, np.float64).T


def abs_scale(xdeq: np.ndarray, wdeq: np.ndarray) -> np.ndarray:
    return np.abs(np.asarray(xdeq, np.float64)) @ np.abs(np.asarray(wdeq, np.float64)).T


def naive_gemm(xdeq: np.ndarray, wdeq: np.ndarray) -> np.ndarray:
    """Triple loop in pure Python (small sizes only), used to pin gemm_ref."""
    M, K = xdeq.shape
    N = wdeq.shape[0]
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(xdeq[m, k]) * float(wdeq[n, k])
            y[m, n] = acc
    return y


def bf16_rne(y: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (8 significant bits, nearest-even) in one rounding step and
    return them as float64.  bf16 subnormals step by 2^-133."""
    y = np.asarray(y, dtype=np.float64)
    m, e = np.frexp(y)                                # y = m * 2**e, |m| in [0.5, 1)
    normal = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    sub = np.ldexp(np.rint(np.ldexp(y, 133)), -133)
    out = np.where(np.abs(y) < 2.0 ** -126, sub, normal)
    return np.where(y == 0, y, out)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |v| (subnormal spacing below 2^-126)."""
    v = np.abs(np.asarray(v, dtype=np.float64))
    _, e = np.frexp(np.where(v == 0, 2.0 ** -126, v))
    return np.ldexp(1.0, np.maximum(e - 8, -133))
