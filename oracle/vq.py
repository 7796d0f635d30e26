"""MXCode PreScale VQ weights and the E4M3-B16 W4A4 layer (oracle; test infrastructure only).

"MXCode: MX-Native Codebook Quantization", abstract and Table 1: PreScale extracts the MX block
scales *before* codebook learning, so the codebook holds pure E2M1 values and a decoded weight
is an MX-native FP4 operand (code x block scale x tensor scale) with no high-precision weight in
between.  Format here (the E4M3-B16-FP4 row of Table 1, with VQ on the input-channel axis,
K = 256 entries of d = 4, one codebook per 64 x 64 QBlock, Figure 3 / appendix Table 4):

  ts_w           FP32 tensor scale  = amax(W) / (6 * 448)
  s_w[n, k/16]   E4M3 block scale   = E4M3_RNE_sat((amax_block / 6) / ts_w)
  v = W / (dec(s_w) * ts_w)          (fp32; 0 where the block scale encodes to 0)
  idx[n, k/4]    index of the nearest codebook entry to v[n, 4j:4j+4] (squared distance, exact
                 in float64; ties to the lowest index)
  W_hat[n, k]    = E2M1(codebook[idx][k % 4]) * dec(s_w) * ts_w

The codebooks themselves are inputs (fit by seeded k-means in the data synthesis; their quality
is not what parity checks).  Bits per weight: 8-bit index per 4 weights = 2.0 BPE of indices
(Figure 2 caption: BPE = log2(K)/d), plus 0.5 BPE of E4M3 scales, plus the codebooks.
"""
from __future__ import annotations

import numpy as np

from . import formats as F
from . import gemm as G
from . import mx


def prescale(w: np.ndarray) -> tuple[np.float32, np.ndarray]:
    """Tensor scale and E4M3 block scales of a weight [N, K] (K % 16 == 0), float32 steps."""
    w32 = np.asarray(w, dtype=np.float32)
    ts = mx.tensor_scale_e4m3(np.abs(w32).max())
    _, sb, ts = mx.quantize_e4m3_b16(w32, ts)
    return ts, sb


def normalized(w: np.ndarray, sb: np.ndarray, ts: np.float32) -> np.ndarray:
    """v = w / (dec(s) * ts) in float32; 0 in blocks whose scale is 0."""
    w32 = np.asarray(w, dtype=np.float32)
    N, K = w32.shape
    S = (F.e4m3_decode(sb).astype(np.float32) * np.float32(ts)).astype(np.float32)
    Sx = np.repeat(S, 16, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (w32 / Sx).astype(np.float32)
    return np.where(Sx == 0, np.float32(0.0), v)


def assign(v: np.ndarray, codebooks: np.ndarray, qn: int = 64, qk: int = 64) -> np.ndarray:
    """Nearest codebook entry per 4-vector along K.  codebooks: [N/qn, K/qk, 256, 4] E2M1 codes.
    Distances are exact in float64 (v is fp32, entries are E2M1), ties go to the lowest index."""
    N, K = v.shape
    QC = K // qk
    cb_vals = F.e2m1_decode(codebooks)                       # [QR, QC, 256, 4]
    idx = np.empty((N, K // 4), dtype=np.uint8)
    v64 = v.astype(np.float64)
    step = 16                                                # QBlocks per numpy batch
    for qr in range(N // qn):
        # points of this row of QBlocks: [QC, qn * qk / 4, 4]
        pts = v64[qr * qn:(qr + 1) * qn].reshape(qn, QC, qk // 4, 4).transpose(1, 0, 2, 3)
        pts = pts.reshape(QC, -1, 4)
        for c0 in range(0, QC, step):
            p = pts[c0:c0 + step]                            # [b, P, 4]
            c = cb_vals[qr, c0:c0 + step]                    # [b, 256, 4]
            d = np.zeros((p.shape[0], p.shape[1], c.shape[1]))
            for i in range(4):                               # exact: squares of fp32 differences
                d += (p[:, :, None, i] - c[:, None, :, i]) ** 2
            best = d.argmin(axis=2)                          # first minimum = lowest index
            blk = best.reshape(-1, qn, qk // 4).transpose(1, 0, 2).reshape(qn, -1)
            idx[qr * qn:(qr + 1) * qn, c0 * qk // 4:(c0 + p.shape[0]) * qk // 4] = blk
    return idx


def decode_codes(idx: np.ndarray, codebooks: np.ndarray, qn: int = 64, qk: int = 64) -> np.ndarray:
    """E2M1 codes [N, K] of the weight the indices select (one nibble per element)."""
    N, K4 = idx.shape
    K = 4 * K4
    qr = (np.arange(N) // qn)[:, None]
    qc = (np.arange(K4) * 4 // qk)[None, :]
    ent = codebooks[qr, qc, idx.astype(np.int64)]            # [N, K/4, 4]
    return ent.reshape(N, K).astype(np.uint8)


def dequant_weight(idx, codebooks, sb, ts, qn=64, qk=64) -> np.ndarray:
    return mx.dequant_e4m3_b16(decode_codes(idx, codebooks, qn, qk), sb, ts)


def pack_codebooks(codebooks: np.ndarray) -> np.ndarray:
    """[QR, QC, 256, 4] nibbles -> [QR, QC, 256, 2] bytes (entry element 2i in the low nibble)."""
    return F.pack_nibbles(codebooks)


def prepare(w: np.ndarray, codebooks: np.ndarray, qn: int = 64, qk: int = 64) -> dict:
    ts, sb = prescale(w)
    idx = assign(normalized(w, sb, ts), codebooks, qn, qk)
    return dict(ts=ts, sb=sb, idx=idx)


def forward(x: np.ndarray, prep: dict, codebooks: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """y = Q_e4m3b16(x) . W_hat^T in float64, and the tolerance scale sum|x_q w_q|."""
    xc, xs, xts = mx.quantize_e4m3_b16(np.asarray(x, dtype=np.float32))
    xd = mx.dequant_e4m3_b16(xc, xs, xts)
    wd = dequant_weight(prep["idx"], codebooks, prep["sb"], prep["ts"])
    return G.gemm_with_scale(xd, wd)


# ------------------------------------------------------------------------------ PostScale
# MXCode abstract: "PostScale, which quantizes learned codebooks to MXFP4".  Reading (the only one
# under which the decoded weight is an MX-native operand, which the abstract requires of all three
# strategies): a QBlock's learned codebook (256 x 4 values, bf16) is quantized with ONE E4M3 block
# scale for the whole codebook, relative to an FP32 tensor scale taken over all codebooks
# (E4M3-B16-FP4 row of Table 1), so that every 16-element block of the decoded weight inside the
# QBlock carries that scale.  The weights are assigned to the nearest quantized entry in value
# space.  No per-weight scales are stored.

def postscale_quantize_codebooks(cent: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.float32]:
    """cent: learned codebooks [QR, QC, 256, 4] (float32-representable values, e.g. bf16).
    Returns (E2M1 codes [QR, QC, 256, 4], E4M3 scale bytes [QR, QC], tensor scale ts), with
    float32 steps as for an E4M3-B16 block: ts = amax(all codebooks) / 2688 (1 if 0);
    s = E4M3((amax(codebook) / 6) / ts); S = dec(s) * ts; code = E2M1(c / S), zero codes where
    S is 0 (sign kept)."""
    c32 = np.asarray(cent, dtype=np.float32)
    QR, QC = c32.shape[:2]
    ts = mx.tensor_scale_e4m3(np.abs(c32).max() if c32.size else 0.0)
    amax = np.abs(c32.reshape(QR, QC, -1)).max(axis=-1).astype(np.float32)
    r = ((amax / np.float32(6.0)).astype(np.float32) / ts).astype(np.float32)
    sb = F.e4m3_encode_nonneg(r.astype(np.float64))
    S = (F.e4m3_decode(sb).astype(np.float32) * ts).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (c32 / S[:, :, None, None]).astype(np.float32)
    q = np.where((S == 0)[:, :, None, None], np.where(np.signbit(c32), -0.0, 0.0), q)
    return F.e2m1_encode(q.astype(np.float64)), sb, ts


def postscale_assign(w: np.ndarray, codes: np.ndarray, sb: np.ndarray, ts: np.float32,
                     qn: int = 64, qk: int = 64) -> np.ndarray:
    """Index of the nearest decoded entry (value e2m1(code) * dec(s_q) * ts, the exact value of
    the MX-native operand) to each 4-vector of W along K.  Squared distances summed over the 4
    coordinates in order, in float64 (entry values are exact in float64); ties go to the lowest
    index."""
    w64 = np.asarray(w, dtype=np.float64)
    N, K = w64.shape
    scale = F.e4m3_decode(sb) * np.float64(np.float32(ts))                      # exact
    vals = F.e2m1_decode(codes) * scale[:, :, None, None]                       # [QR, QC, 256, 4]
    idx = np.empty((N, K // 4), dtype=np.uint8)
    for qr in range(N // qn):
        for qc in range(K // qk):
            p = w64[qr * qn:(qr + 1) * qn, qc * qk:(qc + 1) * qk].reshape(-1, 4)   # row-major
            c = vals[qr, qc]
            d = np.zeros((p.shape[0], c.shape[0]))
            for i in range(4):
                d += (p[:, None, i] - c[None, :, i]) ** 2
            idx[qr * qn:(qr + 1) * qn, qc * qk // 4:(qc + 1) * qk // 4] = \
                d.argmin(axis=1).reshape(qn, qk // 4)
    return idx


def postscale_block_scales(sb_q: np.ndarray, N: int, K: int, qn: int = 64, qk: int = 64) -> np.ndarray:
    """The per-16 E4M3 scale bytes [N, K/16] of the decoded MX-native operand: every block of a
    QBlock carries the QBlock's scale."""
    return np.repeat(np.repeat(sb_q, qn, axis=0), qk // 16, axis=1)[:N, :K // 16]


def postscale_prepare(w: np.ndarray, cent: np.ndarray, qn: int = 64, qk: int = 64) -> dict:
    codes, sbq, ts = postscale_quantize_codebooks(cent)
    idx = postscale_assign(w, codes, sbq, ts, qn, qk)
    return dict(codes=codes, sbq=sbq, ts=ts, idx=idx)


def postscale_forward(x: np.ndarray, prep: dict) -> tuple[np.ndarray, np.ndarray]:
    """y = Q_e4m3b16(x) . W_hat^T, W_hat[n,k] = e2m1(code) * dec(s_q) * ts; float64."""
    from . import gemm as G
    N, K4 = prep["idx"].shape
    sb = postscale_block_scales(prep["sbq"], N, 4 * K4)
    xc, xs, xts = mx.quantize_e4m3_b16(np.asarray(x, dtype=np.float32))
    xd = mx.dequant_e4m3_b16(xc, xs, xts)
    wd = mx.dequant_e4m3_b16(decode_codes(prep["idx"], prep["codes"]), sb, prep["ts"])
    return G.gemm_with_scale(xd, wd)


# ------------------------------------------------------------------------------ PreScale+
# MXCode abstract: "PreScale+, which further compresses these scales using VQ"; appendix Table 4
# caption: "PreScale+ compresses scales using Ks=256, ds=8".  Reading: the E4M3 block scales of
# PreScale are grouped 8 at a time along K (one row, 8 x 16 = 128 weights per group); each group
# is replaced by the nearest of Ks = 256 scale vectors of a per-tensor scale codebook (distance
# between decoded scale values, squared, summed in order in float64; ties to the lowest index);
# the weight is then normalised by the compressed scales and assigned as in PreScale.

def prescale_plus_assign_scales(sb: np.ndarray, scb: np.ndarray, ds: int = 8) -> np.ndarray:
    """sb: E4M3 scale bytes [N, K/16]; scb: scale codebook [Ks, ds] E4M3 bytes.
    Returns scale indices [N, K/16/ds] (uint8)."""
    v = F.e4m3_decode(sb).astype(np.float64)
    N, G16 = v.shape
    grp = v.reshape(N, G16 // ds, ds)
    c = F.e4m3_decode(scb).astype(np.float64)                 # [Ks, ds]
    d = np.zeros((N, G16 // ds, c.shape[0]))
    for i in range(ds):
        d += (grp[:, :, None, i] - c[None, None, :, i]) ** 2
    return d.argmin(axis=2).astype(np.uint8)


def prescale_plus_scales(sidx: np.ndarray, scb: np.ndarray) -> np.ndarray:
    """The compressed scale bytes [N, K/16]: scb[sidx[n, g]][i] for block 8g + i."""
    N, Gs = sidx.shape
    return scb[sidx.astype(np.int64)].reshape(N, Gs * scb.shape[1])


def prescale_plus_prepare(w: np.ndarray, codebooks: np.ndarray, scb: np.ndarray,
                          qn: int = 64, qk: int = 64, ds: int = 8) -> dict:
    ts, sb = prescale(w)
    sidx = prescale_plus_assign_scales(sb, scb, ds)
    sb2 = prescale_plus_scales(sidx, scb)
    idx = assign(normalized(w, sb2, ts), codebooks, qn, qk)
    return dict(ts=ts, sb=sb2, sidx=sidx, idx=idx)
