"""Block quantizers (oracle; test infrastructure only).

quantize_e8m0_b32 -- MXFP4 with an E8M0 shared exponent per 32 elements along K, the OCP
    Microscaling rule the PRQuant page quantizes activations and weights with ("MXFP4",
    §4 Method and "Kernel design for efficient inference"): shared exponent
    floor(log2 amax) - 2 (2 = the largest E2M1 exponent), elements x / 2^e rounded to
    nearest-even E2M1 and saturated at +-6.
quantize_e4m3_b16 -- E4M3-B16-FP4 with an FP32 tensor scale (MXCode, Table 1, row
    "E4M3-B16-FP4"): the block scale targets amax/6, expressed relative to a tensor scale
    amax_T/(6*448) so that it fits E4M3.  Every step is an IEEE float32 operation in the
    order written, so the GPU takes the same integer decisions.
quantize_int4_g128 -- symmetric INT4 per (row, 128-group) with an fp32 scale amax/7
    (MosaicQuant, "Dense Base and Sparse Residuals"; granularity is a reading, the page
    does not state it).
"""
from __future__ import annotations

import numpy as np

from . import formats as F


def mx_shared_exponent(amax: np.ndarray) -> np.ndarray:
    """floor(log2 amax) - 2, clamped to [-127, 127]; amax == 0 gives -127."""
    amax = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(amax)                  # amax = m * 2**ex with m in [0.5, 1)
    e = ex.astype(np.int64) - 1 - 2
    e = np.where(amax == 0, -127, e)
    return np.clip(e, -127, 127)


def quantize_e8m0_b32(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """x float64 [R, K] (K % 32 == 0) -> (codes uint8 [R, K] one nibble per byte,
    scale bytes uint8 [R, K/32])."""
    x = np.asarray(x, dtype=np.float64)
    R, K = x.shape
    assert K % 32 == 0
    blocks = x.reshape(R, K // 32, 32)
    e = mx_shared_exponent(np.abs(blocks).max(axis=-1))
    scaled = blocks * np.ldexp(1.0, -e)[..., None]          # exact: power-of-two scaling
    codes = F.e2m1_encode(scaled).reshape(R, K)
    return codes, (e + 127).astype(np.uint8)


def quantize_e8m0_b32_searched(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """MXFP4 with a local search of the E8M0 block scale (PRQuant §5.3, "PRQuant (E8M0-W)": a
    weight-side local block-scale search).  Reading: per 32-block the candidates are the OCP
    exponent e0 = floor(log2 amax) - 2 and its neighbours e0 + 1 and e0 - 1 (clamped to
    [-127, 127]); each is applied with the same element rule (RNE to E2M1, saturating at 6) and
    the block keeps the one with the smallest sum of squared errors (float64, summed over the 32
    elements in order), trying e0, then e0 + 1, then e0 - 1, a later one only if strictly
    better.  Same outputs as quantize_e8m0_b32."""
    x = np.asarray(x, dtype=np.float64)
    R, K = x.shape
    assert K % 32 == 0
    blocks = x.reshape(R, K // 32, 32)
    e0 = mx_shared_exponent(np.abs(blocks).max(axis=-1))
    best_e = e0.copy()
    best_codes = F.e2m1_encode(blocks * np.ldexp(1.0, -e0)[..., None])
    best_err = _block_sq_err(blocks, best_codes, e0)
    for de in (1, -1):
        e = np.clip(e0 + de, -127, 127)
        codes = F.e2m1_encode(blocks * np.ldexp(1.0, -e)[..., None])
        err = _block_sq_err(blocks, codes, e)
        better = err < best_err
        best_e = np.where(better, e, best_e)
        best_codes = np.where(better[..., None], codes, best_codes)
        best_err = np.where(better, err, best_err)
    return best_codes.reshape(R, K).astype(np.uint8), (best_e + 127).astype(np.uint8)


def _block_sq_err(blocks: np.ndarray, codes: np.ndarray, e: np.ndarray) -> np.ndarray:
    d = blocks - F.e2m1_decode(codes) * np.ldexp(1.0, e)[..., None]
    acc = np.zeros(blocks.shape[:-1])
    for i in range(blocks.shape[-1]):                   # summed in element order
        acc += d[..., i] * d[..., i]
    return acc


def dequant_e8m0_b32(codes: np.ndarray, sbytes: np.ndarray) -> np.ndarray:
    R, K = codes.shape
    v = F.e2m1_decode(codes).reshape(R, K // 32, 32)
    return (v * F.e8m0_decode(sbytes)[..., None]).reshape(R, K)


def tensor_scale_e4m3(amax_t: float) -> np.float32:
    """FP32 tensor scale amax_T / (6*448), or 1 for an all-zero tensor."""
    a = np.float32(amax_t)
    if a == 0:
        return np.float32(1.0)
    return np.float32(a / np.float32(2688.0))


def quantize_e4m3_b16(x: np.ndarray, ts: np.float32 | None = None
                      ) -> tuple[np.ndarray, np.ndarray, np.float32]:
    """x [R, K] of float32-representable values (K % 16 == 0) ->
    (codes [R, K] nibbles, E4M3 scale bytes [R, K/16], tensor scale fp32).

    Steps (float32 each):  ts = amax_T / 2688;  t = amax_b / 6;  s = E4M3(t / ts) RNE, satfinite;
    S = dec(s) * ts;  code = E2M1(x / S).  A block whose scale encodes to 0 gets all-zero codes
    (sign kept).  ``ts`` may be passed in (weights carry their own).
    """
    x32 = np.asarray(x, dtype=np.float32)
    R, K = x32.shape
    assert K % 16 == 0
    if ts is None:
        ts = tensor_scale_e4m3(np.abs(x32).max() if x32.size else 0.0)
    ts = np.float32(ts)
    blocks = x32.reshape(R, K // 16, 16)
    amax_b = np.abs(blocks).max(axis=-1).astype(np.float32)
    t = (amax_b / np.float32(6.0)).astype(np.float32)
    r = (t / ts).astype(np.float32)
    sb = F.e4m3_encode_nonneg(r.astype(np.float64))
    S = (F.e4m3_decode(sb).astype(np.float32) * ts).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (blocks / S[..., None]).astype(np.float32)
    q = np.where((S == 0)[..., None], np.where(np.signbit(blocks), -0.0, 0.0), q)
    codes = F.e2m1_encode(q.astype(np.float64)).reshape(R, K)
    return codes, sb, ts


def dequant_e4m3_b16(codes: np.ndarray, sbytes: np.ndarray, ts: float) -> np.ndarray:
    """Exact value of each element: code * dec(s) * ts, in float64 (the product of the two
    scales is not rounded to float32 here; it is the real number the format denotes)."""
    R, K = codes.shape
    v = F.e2m1_decode(codes).reshape(R, K // 16, 16)
    s = F.e4m3_decode(sbytes) * np.float64(np.float32(ts))
    return (v * s[..., None]).reshape(R, K)


def quantize_int4_g128(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """x [R, K] float32-representable (K % 128 == 0) -> (q int64 [R, K] in [-7, 7],
    scales float32 [R, K/128]).  s = amax / 7 (fp32); q = clamp(rint_even(x / s), -7, 7);
    an all-zero group has s = 0 and q = 0."""
    x32 = np.asarray(x, dtype=np.float32)
    R, K = x32.shape
    assert K % 128 == 0
    g = x32.reshape(R, K // 128, 128)
    s = (np.abs(g).max(axis=-1) / np.float32(7.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (g / s[..., None]).astype(np.float32)
    r = np.where((s == 0)[..., None], np.float32(0.0), r)
    q = np.clip(np.rint(r.astype(np.float64)), -7, 7).astype(np.int64)   # rint: ties to even
    return q.reshape(R, K), s
