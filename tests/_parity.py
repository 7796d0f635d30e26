"""Shared helpers for the parity tests: tolerance checks against the oracle (test-only)."""
import numpy as np

from oracle import gemm as G

REL_TOL = 1e-5   # |y32 - y_ref| <= 1e-5 * sum_k |x_q w_q|, per element, before the bf16 cast


def check_fp32(y32: np.ndarray, y_ref: np.ndarray, t: np.ndarray, what: str = "") -> float:
    """Returns the worst ratio |y32 - y_ref| / (1e-5 * t); fails if it exceeds 1."""
    err = np.abs(y32.astype(np.float64) - y_ref)
    bound = REL_TOL * t
    bad = err > bound
    worst = float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} elements outside 1e-5*sum|xw|; worst ratio {worst:.3g}"
    return worst


def check_bf16(y_bf16: np.ndarray, y_ref: np.ndarray, t: np.ndarray, what: str = "") -> None:
    """bf16 output within 1 ulp of bf16_RNE(y_ref), widened by the fp32 bound 1e-5 * sum|x w|
    (which only matters where cancellation makes y_ref small against sum|x w|): a correctly
    rounded cast of any y32 that passes check_fp32 lands inside this."""
    ref = G.bf16_rne(y_ref)
    err = np.abs(y_bf16.astype(np.float64) - ref)
    allow = G.bf16_ulp(ref) + REL_TOL * t
    bad = err > allow
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} bf16 outputs beyond 1 ulp"
