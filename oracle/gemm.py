"""W4A4 GEMM reference (oracle; test infrastructure only).

y[m, n] = sum_k deq(x)[m, k] * deq(w)[n, k] in float64, the plain definition of the quantized
linear layer y = X W^T that all five pages share (PRQuant, §4 "Kernel design for efficient
inference": one MXFP4 GEMM over the quantized operands; MXCode abstract: MX-native W4A4
operands).  The dequantized operands are exact in float64, each product is exact, and the
float64 sum is within K * 2^-53 relative of the exact sum, far inside the float tolerance.

The sum itself is a plain C loop (``gemm_sum.c``): one running float64 total per element, terms
added in ascending k, no blocking and no library matmul, so its rounding order is the one written
here and not a BLAS kernel's.  The C file is compiled with gcc on first use (or by the package's
build step) into ``oracle/_build/``; it shares nothing with the CUDA library.

The tolerance scale t[m, n] = sum_k |deq x[m,k] * deq w[n,k]| bounds an fp32-accumulated
result: |y_gpu - y| <= 1e-5 * t per element before the bf16 cast.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gemm_sum.c")
_LIB = os.path.join(_HERE, "_build", "liboracle_gemm.so")
_lib = None


def build_c(force: bool = False) -> str:
    """Compile gemm_sum.c (gcc, -O2, OpenMP, no fused multiply-add) if it is newer than the
    library; return the library path."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = f"{_LIB}.{os.getpid()}.tmp"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared",
                    "-fPIC", "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _c():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build_c())
        L.oracle_gemm_nt.restype = None
        L.oracle_gemm_nt.argtypes = [ctypes.c_int64] * 3 + [ctypes.c_void_p] * 4
        _lib = L
    return _lib


def gemm_with_scale(xdeq: np.ndarray, wdeq: np.ndarray, want_scale: bool = True):
    """(y, t): y = sum_k x[m,k] w[n,k] and t = sum_k |x[m,k] w[n,k]|, each summed in ascending k
    in float64.  x [M, K], w [N, K]."""
    x = np.ascontiguousarray(xdeq, dtype=np.float64)
    w = np.ascontiguousarray(wdeq, dtype=np.float64)
    assert x.ndim == 2 and w.ndim == 2 and x.shape[1] == w.shape[1]
    M, K = x.shape
    N = w.shape[0]
    y = np.empty((M, N))
    t = np.empty((M, N)) if want_scale else None
    if M and N:
        _c().oracle_gemm_nt(M, N, K, x.ctypes.data, w.ctypes.data, y.ctypes.data,
                            t.ctypes.data if t is not None else None)
    return y, t


def gemm_ref(xdeq: np.ndarray, wdeq: np.ndarray) -> np.ndarray:
    return gemm_with_scale(xdeq, wdeq, want_scale=False)[0]


def abs_scale(xdeq: np.ndarray, wdeq: np.ndarray) -> np.ndarray:
    return gemm_with_scale(xdeq, wdeq)[1]


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
