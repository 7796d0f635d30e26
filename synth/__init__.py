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
    "activations_bf16", "student_t", "uniform_nibble_bytes", "uniform_bytes", "vq_raw_codebooks",
    "scale_codebook",
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


_E2M1_GRID = np.array([-6.0, -4.0, -3.0, -2.0, -1.5, -1.0, -0.5, 0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
_E2M1_CODE = np.array([15, 14, 13, 12, 11, 10, 9, 0, 1, 2, 3, 4, 5, 6, 7], dtype=np.uint8)


def vq_codebooks(seed: int, w: np.ndarray, qn: int = 64, qk: int = 64, entries: int = 256,
                 iters: int = 4, chunk: int = 128) -> np.ndarray:
    """Synthesize one FP4 codebook per qn x qk QBlock by seeded k-means (data synthesis only).

    Each 4-vector along K is first brought to the E2M1 range by its 16-block's amax / 6 (a
    generator-side normalisation in float64, not the method's E4M3 scale), then k-means with
    `entries` centroids (distinct random points as the initial centroids, `iters` Lloyd steps) runs
    per QBlock, and each centroid coordinate snaps to the closest signed E2M1 grid value.
    Returns E2M1 codes [N/qn, K/qk, entries, 4] (uint8 nibbles).
    """
    g = rng(seed * 31 + 7)
    N, K = w.shape
    QR, QC = N // qn, K // qk
    blk = np.abs(w.reshape(N, K // 16, 16)).max(-1, keepdims=True)
    v = (w.reshape(N, K // 16, 16) / np.where(blk == 0, 1.0, blk / 6.0)).reshape(N, K)
    # points per QBlock: [QR*QC, qn*qk/4, 4]
    pts = v.reshape(QR, qn, QC, qk // 4, 4).transpose(0, 2, 1, 3, 4).reshape(QR * QC, -1, 4)
    out = np.empty((QR * QC, entries, 4), dtype=np.uint8)
    P = pts.shape[1]
    for c0 in range(0, QR * QC, chunk):
        p = pts[c0:c0 + chunk].astype(np.float32)                      # [B, P, 4]
        B = p.shape[0]
        init = np.stack([g.choice(P, entries, replace=False) for _ in range(B)])
        cent = np.take_along_axis(p, init[:, :, None], axis=1)        # [B, E, 4]
        for _ in range(iters):
            d = (p * p).sum(-1)[:, :, None] - 2 * p @ cent.transpose(0, 2, 1) + \
                (cent * cent).sum(-1)[:, None, :]
            lab = d.argmin(-1)                                         # [B, P]
            flat = (lab + np.arange(B)[:, None] * entries).reshape(-1)
            sums = np.zeros((B * entries, 4), np.float64)
            np.add.at(sums, flat, p.reshape(-1, 4))
            cnt = np.bincount(flat, minlength=B * entries).astype(np.float64)
            newc = (sums / np.maximum(cnt, 1)[:, None]).reshape(B, entries, 4).astype(np.float32)
            cent = np.where((cnt == 0).reshape(B, entries, 1), cent, newc)
        snap = np.abs(cent[..., None] - _E2M1_GRID).argmin(-1)
        out[c0:c0 + B] = _E2M1_CODE[snap]
    return out.reshape(QR, QC, entries, 4)


def vq_raw_codebooks(seed: int, w: np.ndarray, qn: int = 64, qk: int = 64, entries: int = 256,
                     iters: int = 4, chunk: int = 128) -> np.ndarray:
    """Learned codebooks in value space (bf16 centroids), one per qn x qk QBlock, by seeded
    k-means on the raw 4-vectors along K (data synthesis only; the method then quantizes them).
    Returns float32 [N/qn, K/qk, entries, 4] holding bf16 values."""
    g = rng(seed * 37 + 11)
    N, K = w.shape
    QR, QC = N // qn, K // qk
    pts = np.asarray(w, np.float64).reshape(QR, qn, QC, qk // 4, 4).transpose(0, 2, 1, 3, 4)
    pts = pts.reshape(QR * QC, -1, 4)
    out = np.empty((QR * QC, entries, 4), dtype=np.float32)
    P = pts.shape[1]
    for c0 in range(0, QR * QC, chunk):
        p = pts[c0:c0 + chunk].astype(np.float32)
        B = p.shape[0]
        init = np.stack([g.choice(P, entries, replace=False) for _ in range(B)])
        cent = np.take_along_axis(p, init[:, :, None], axis=1)
        for _ in range(iters):
            d = (p * p).sum(-1)[:, :, None] - 2 * p @ cent.transpose(0, 2, 1) + \
                (cent * cent).sum(-1)[:, None, :]
            lab = d.argmin(-1)
            flat = (lab + np.arange(B)[:, None] * entries).reshape(-1)
            sums = np.zeros((B * entries, 4), np.float64)
            np.add.at(sums, flat, p.reshape(-1, 4))
            cnt = np.bincount(flat, minlength=B * entries).astype(np.float64)
            newc = (sums / np.maximum(cnt, 1)[:, None]).reshape(B, entries, 4).astype(np.float32)
            cent = np.where((cnt == 0).reshape(B, entries, 1), cent, newc)
        out[c0:c0 + B] = cent
    bits = to_bf16_bits(out)
    return bf16_bits_to_f64(bits).astype(np.float32).reshape(QR, QC, entries, 4)


def scale_codebook(seed: int, sb: np.ndarray, entries: int = 256, ds: int = 8,
                   iters: int = 6) -> np.ndarray:
    """A per-tensor codebook of `entries` scale vectors of length ds (E4M3 bytes) for groups of ds
    consecutive block scales along K: seeded k-means on the scale bytes of the groups, rounded to
    the nearest byte (data synthesis only).  sb: E4M3 scale bytes [N, K/16]."""
    g = rng(seed * 41 + 3)
    pts = np.asarray(sb, np.float64).reshape(-1, ds)
    uniq = np.unique(pts, axis=0)
    if len(uniq) <= entries:
        out = np.zeros((entries, ds), np.uint8)
        out[:len(uniq)] = uniq.astype(np.uint8)
        return out
    cent = uniq[g.choice(len(uniq), entries, replace=False)]
    for _ in range(iters):
        d = (pts * pts).sum(-1)[:, None] - 2 * pts @ cent.T + (cent * cent).sum(-1)[None, :]
        lab = d.argmin(-1)
        sums = np.zeros((entries, ds))
        np.add.at(sums, lab, pts)
        cnt = np.bincount(lab, minlength=entries).astype(np.float64)
        cent = np.where(cnt[:, None] > 0, sums / np.maximum(cnt, 1)[:, None], cent)
    return np.clip(np.rint(cent), 0, 126).astype(np.uint8)


def zipf_router_logits(seed: int, T: int, E: int = 128, s: float = 1.1) -> np.ndarray:
    """Router logits [T, E] fp32 for a Zipf(s) expert popularity: p_e ~ r_e^-s with r a seeded
    permutation of the ranks 1..E; logit = ln p_e + Gumbel(0, 1) noise, so that the top-k of a
    token is a Gumbel-top-k draw from p without replacement."""
    g = rng(seed * 13 + 5)
    ranks = g.permutation(E) + 1.0
    p = ranks ** -s
    p /= p.sum()
    u = g.random((T, E))
    u = np.clip(u, 1e-300, 1.0 - 1e-16)
    return (np.log(p)[None, :] - np.log(-np.log(u))).astype(np.float32)


def cluster_rows(seed: int, rows: int, K: int, nu: float = 4.0, C: int = 16,
                 iters: int = 6) -> tuple[np.ndarray, np.ndarray]:
    """Per-row C-centroid codebooks fit by 1-D k-means (Lloyd, quantile start) on Student-t(nu)
    weights [rows, K] (data synthesis only).  Returns (centroids as bf16 bits [rows, C], ascending;
    4-bit indices [rows, K] of the nearest bf16 centroid, ties to the lower index)."""
    w = student_t(seed, (rows, K), nu).astype(np.float64)
    srt = np.sort(w, axis=1)
    lo, hi = srt[:, :1], srt[:, -1:]
    span = float((hi - lo).max()) * 2.0 + 1.0
    key = (np.arange(rows)[:, None] * span + (srt - lo)).reshape(-1)     # row-major ascending
    cs = np.concatenate([np.zeros((rows, 1)), np.cumsum(srt, axis=1)], axis=1)
    q = (np.arange(C) + 0.5) / C
    cent = srt[:, np.minimum((q * K).astype(int), K - 1)]
    rows_off = np.arange(rows)[:, None]
    for _ in range(iters):
        mids = 0.5 * (cent[:, 1:] + cent[:, :-1])
        pos = np.searchsorted(key, (rows_off * span + (mids - lo)).reshape(-1), side="left")
        pos = pos.reshape(rows, C - 1) - rows_off * K
        b = np.concatenate([np.zeros((rows, 1), int), pos, np.full((rows, 1), K)], axis=1)
        cnt = np.diff(b, axis=1)
        sums = np.take_along_axis(cs, b[:, 1:], 1) - np.take_along_axis(cs, b[:, :-1], 1)
        cent = np.where(cnt > 0, sums / np.maximum(cnt, 1), cent)
        cent = np.sort(cent, axis=1)
    cbits = to_bf16_bits(cent)
    cq = bf16_bits_to_f64(cbits)
    order = np.argsort(cq, axis=1, kind="stable")
    cbits = np.take_along_axis(cbits, order, 1)
    cq = np.take_along_axis(cq, order, 1)
    # nearest centroid in the original order: number of midpoints strictly below the value
    mids = 0.5 * (cq[:, 1:] + cq[:, :-1])
    lo2 = np.minimum(w.min(axis=1, keepdims=True), cq[:, :1])
    span2 = float((np.maximum(w.max(axis=1, keepdims=True), cq[:, -1:]) - lo2).max()) * 2.0 + 1.0
    mkey = (rows_off * span2 + (mids - lo2)).reshape(-1)
    idx = np.searchsorted(mkey, (rows_off * span2 + (w - lo2)).reshape(-1), side="left")
    idx = idx.reshape(rows, K) - rows_off * (C - 1)
    return cbits, np.clip(idx, 0, C - 1).astype(np.uint8)
