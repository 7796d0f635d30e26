"""Online block-Hadamard rotation before activation quantization (oracle; test infrastructure only).

CodeQuant, accuracy tables (Table 2 and appendix Table 8): the "had" variants enable "online
Hadamard transforms during the quantization process".  The pages give no size or algorithm;
readings:
  * the transform is block-diagonal with Sylvester Hadamard blocks of b = 32 (the MX block), so
    that every quantization block is rotated on its own and no block mixes with another;
  * the activation side is unnormalised: x' = x . blockdiag(H_b), computed in float32 by the fast
    Walsh-Hadamard butterfly in the order h = 1, 2, 4, 8, 16, each step (a, b) -> (a + b, a - b)
    an IEEE float32 addition or subtraction (so the quantized codes of x' are reproducible bit for
    bit); x' is then quantized by the layer's activation rule;
  * the weight is rotated offline, W' = W . blockdiag(H_b) / b (exact in float64: b is a power of
    two), so that x' W'^T = x H H^T W^T / b = x W^T.
"""
from __future__ import annotations

import numpy as np


def sylvester(n: int) -> np.ndarray:
    """Unnormalised Hadamard matrix of order n (a power of two): H_1 = [1],
    H_2m = [[H_m, H_m], [H_m, -H_m]]; entries +-1 (int64)."""
    assert n >= 1 and n & (n - 1) == 0
    h = np.ones((1, 1), dtype=np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def rotate_activation_f32(x: np.ndarray, b: int = 32) -> np.ndarray:
    """x' = x . blockdiag(H_b) along the last axis, in float32 by the butterfly (h = 1, 2, ...,
    b/2; (a, b) -> (a + b, a - b)).  x: float32-representable values [..., K], K % b == 0, whose
    rotated blocks stay finite in float32."""
    v = np.array(x, dtype=np.float32, copy=True)
    K = v.shape[-1]
    assert K % b == 0
    blk = v.reshape(v.shape[:-1] + (K // b, b))
    h = 1
    while h < b:
        g = blk.reshape(blk.shape[:-1] + (b // (2 * h), 2, h))
        lo = g[..., 0, :].copy()
        hi = g[..., 1, :].copy()
        g[..., 0, :] = (lo + hi).astype(np.float32)
        g[..., 1, :] = (lo - hi).astype(np.float32)
        blk = g.reshape(blk.shape)
        h *= 2
    return blk.reshape(v.shape)


def rotate_weight(w: np.ndarray, b: int = 32) -> np.ndarray:
    """W' = W . blockdiag(H_b) / b along K in float64 (a matmul): exact while the b values of a
    block, bf16 or fp32, span few enough binary orders that their sum fits 53 bits; otherwise
    rounded by the float64 sums."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    H = sylvester(b).astype(np.float64)
    return (w.reshape(N, K // b, b) @ H).reshape(N, K) / b
