"""Number-format codecs, written as plain definitions (oracle; test infrastructure only).

E2M1, E8M0, E4M3 and UE5M3 follow MXCode (MX-Native Codebook Quantization), Table 1
("Block-scaled FP4 formats compared in this work"; all use E2M1 elements and 8-bit block
scales), and the OCP Microscaling formats specification that the PRQuant page cites for
MXFP4/NVFP4.  Encoders are "nearest representable value, ties to the even code", found by
searching the whole value table, so that they are checkable by eye against the table.
"""
from __future__ import annotations

import numpy as np

# --- E2M1 (FP4) ------------------------------------------------------------------------
# 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; magnitude codes 0..7.
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit codes (uint8 values 0..15) -> float64; bit 3 is the sign."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where(c & 8, -mag, mag)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Round to the nearest E2M1 value, ties to the even magnitude code, saturating at 6.

    The sign bit copies the sign of the input (IEEE style), so negative values that round to
    zero (and -0.0) give code 0x8.  Input must be finite.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    flat, res = v.reshape(-1), out.reshape(-1)
    step = 1 << 20                                         # bounded temporaries
    for i in range(0, flat.size, step):
        c = flat[i:i + step]
        a = np.minimum(np.abs(c), 6.0)                     # saturate at the largest magnitude
        d = np.abs(a[:, None] - E2M1_MAGNITUDES)           # distance to each magnitude
        tied = d == d.min(axis=-1, keepdims=True)
        # among the nearest magnitudes prefer an even code; codes ascend with magnitude
        even = tied & ((np.arange(8) & 1) == 0)
        code = np.where(even.any(-1), even.argmax(-1), tied.argmax(-1)).astype(np.uint8)
        res[i:i + step] = code | (np.signbit(c).astype(np.uint8) << 3)
    return out


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., 2j] goes to the low nibble and [..., 2j+1] to the high nibble of byte j."""
    c = np.asarray(codes, dtype=np.uint8)
    assert c.shape[-1] % 2 == 0
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


# --- E8M0 (shared power-of-two block scale) -------------------------------------------
def e8m0_decode(b: np.ndarray) -> np.ndarray:
    """Biased exponent byte -> 2**(b-127).  0xFF is the NaN encoding and is rejected."""
    b = np.asarray(b).astype(np.int64)
    if np.any(b == 255):
        raise ValueError("E8M0 byte 0xFF is NaN")
    return np.ldexp(1.0, b - 127)


# --- E4M3 (OCP FP8 E4M3, finite-only "fn" variant) --------------------------------------
def _e4m3_table() -> np.ndarray:
    """Value of every byte 0..255 (NaN for S.1111.111)."""
    vals = np.empty(256)
    for byte in range(256):
        s, e, m = byte >> 7, (byte >> 3) & 0xF, byte & 7
        if e == 0xF and m == 7:
            vals[byte] = np.nan
            continue
        if e == 0:
            mag = (m / 8.0) * 2.0 ** (1 - 7)            # subnormal
        else:
            mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
        vals[byte] = -mag if s else mag
    return vals


E4M3_TABLE = _e4m3_table()
E4M3_MAX = 448.0


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(b).astype(np.int64) & 0xFF]


def e4m3_encode_nonneg(v: np.ndarray) -> np.ndarray:
    """Unsigned E4M3 scale encode: nearest of the 127 finite non-negative values, ties to even
    code, values above 448 saturate to 448 (satfinite).  Input must be finite and >= 0."""
    v = np.asarray(v, dtype=np.float64)
    assert np.all(v >= 0) and np.all(np.isfinite(v))
    table = E4M3_TABLE[:127]                          # bytes 0x00..0x7E, ascending
    out = np.empty(v.shape, dtype=np.uint8)
    flat, res = v.reshape(-1), out.reshape(-1)
    # nearest by bisection on the sorted table, then the tie rule
    hi = np.searchsorted(table, flat, side="left").clip(1, 126)
    lo = hi - 1
    dlo, dhi = flat - table[lo], table[hi] - flat
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(flat >= table[126], 126, code)       # satfinite
    res[:] = code.astype(np.uint8)
    return out


# --- UE5M3 (unsigned, 5 exponent bits bias 15, 3 mantissa bits; all-ones mantissa at the top
# exponent reserved) -- closed form only, the MXCode appendix evaluates it by emulation --------
def ue5m3_decode(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b).astype(np.int64) & 0xFF
    e, m = b >> 3, b & 7
    sub = (m / 8.0) * 2.0 ** (1 - 15)
    nor = (1.0 + m / 8.0) * 2.0 ** (e - 15)
    out = np.where(e == 0, sub, nor)
    return np.where((e == 31) & (m == 7), np.nan, out)


# --- INT4 (symmetric, codes -7..7 stored as two's-complement nibbles) ---------------------
def int4_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes).astype(np.int64) & 0xF
    return np.where(c >= 8, c - 16, c).astype(np.int64)


def int4_encode(q: np.ndarray) -> np.ndarray:
    q = np.asarray(q).astype(np.int64)
    assert np.all(np.abs(q) <= 7)
    return (q & 0xF).astype(np.uint8)


# --- bf16 ---------------------------------------------------------------------------------
def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact: the upper half of an IEEE binary32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
