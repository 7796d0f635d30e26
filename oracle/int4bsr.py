"""INT4 dense base + block-sparse INT4 residual (oracle; test infrastructure only).

MosaicQuant ("Inlier-Outlier Disaggregation for Unified 4-Bit LLM Quantization"), "Dense Base and
Sparse Residuals": W = dense 4-bit base + a few sparse 4-bit residual blocks; "Activation-aware
Delta-Hessian Block Selection": residual blocks are scored by the reduction in squared error
weighted by calibration-activation sensitivity and the Top-K are kept; "ZipperEngine": both
branches are computed in one fused GEMM.  The page gives no formulas; the readings here:

  base      per (row n, 128-group g): sw = fp16(amax / 7) (fp32 divide, RNE to fp16),
            q = clamp(rint(w / sw), -7, 7) (fp32 divide, ties to even), 0 when sw == 0
  delta     dW = W - q * sw                       (float64, exact)
  score     of the 16 x 128 block (nb, g): sum over its 16 rows, then 128 columns, of
            abar_k * |dW[n, k]|, abar_k = mean_t |x[t, k]| over the calibration rows; both sums
            are taken sequentially in that order (float64)
  select    the round(density * blocks) largest scores, ties to the lower block id nb*(K/128)+g
  residual  each selected block's rows are quantized like the base, on fp32(dW):
            sr = fp16(amax / 7), r = clamp(rint(dW / sr), -7, 7)
  activation per (token m, 128-group g): sx = amax / 7 (fp32), qx = clamp(rint(x / sx), -7, 7)
  forward   y[m, n] = sum_g sx[m,g] sw[n,g] I_g[m,n] + sum_{(nb(n),g) selected} sx[m,g] sr[n,g] R_g[m,n]
            with I_g, R_g the exact integer dot products over the group.
"""
from __future__ import annotations

import numpy as np

from . import gemm as G
from . import mx


def quant_rows_g128(w32: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric INT4 per (row, 128-group) with fp16 scales.  w32 float32 [R, K]."""
    R, K = w32.shape
    g = w32.reshape(R, K // 128, 128)
    s32 = (np.abs(g).max(axis=-1) / np.float32(7.0)).astype(np.float32)
    s16 = s32.astype(np.float16)
    sf = s16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (g / sf[..., None]).astype(np.float32)
    r = np.where((sf == 0)[..., None], np.float32(0.0), r)
    q = np.clip(np.rint(r.astype(np.float64)), -7, 7).astype(np.int64)
    return q.reshape(R, K), s16


def dequant_rows(q: np.ndarray, s16: np.ndarray) -> np.ndarray:
    R, K = q.shape
    return (q.reshape(R, K // 128, 128) * s16.astype(np.float64)[..., None]).reshape(R, K)


def abar(x_calib: np.ndarray) -> np.ndarray:
    """mean_t |x[t, k]|, summed over t in order (float64)."""
    acc = np.zeros(x_calib.shape[1])
    for t in range(x_calib.shape[0]):
        acc += np.abs(x_calib[t])
    return acc / x_calib.shape[0]


def block_scores(dw: np.ndarray, a: np.ndarray, bn: int = 16, bk: int = 128) -> np.ndarray:
    """Scores [N/bn, K/bk]: sequential sum over the block's rows then columns of a_k |dW|."""
    N, K = dw.shape
    p = np.abs(dw) * a[None, :]
    p = p.reshape(N // bn, bn, K // bk, bk).transpose(0, 2, 1, 3).reshape(N // bn, K // bk, bn * bk)
    return np.cumsum(p, axis=2)[:, :, -1]


def prepare(w: np.ndarray, x_calib: np.ndarray, density: float = 0.02, bn: int = 16,
            bk: int = 128) -> dict:
    """Offline preparation.  w: bf16 values as float64 [N, K]; x_calib: bf16 values [T, K]."""
    N, K = w.shape
    w32 = w.astype(np.float32)
    q, sw = quant_rows_g128(w32)
    dw = w - dequant_rows(q, sw)
    sc = block_scores(dw, abar(x_calib), bn, bk)
    nblk = sc.size
    keep = int(round(density * nblk))
    flat = sc.reshape(-1)
    order = sorted(range(nblk), key=lambda i: (-flat[i], i))[:keep]
    sel = np.array(sorted(order), dtype=np.int64)            # ascending block id = (nb, g) order
    nb_of, g_of = sel // (K // bk), sel % (K // bk)
    rows = []
    for nb, g in zip(nb_of, g_of):
        rows.append(dw[nb * bn:(nb + 1) * bn, g * bk:(g + 1) * bk].astype(np.float32))
    if rows:
        rq, rs = quant_rows_g128(np.concatenate(rows, axis=0))
        rq = rq.reshape(keep, bn, bk)
        rs = rs.reshape(keep, bn)
    else:
        rq = np.zeros((0, bn, bk), np.int64)
        rs = np.zeros((0, bn), np.float16)
    rowptr = np.zeros(N // bn + 1, np.int64)
    np.add.at(rowptr, nb_of + 1, 1)
    rowptr = np.cumsum(rowptr)
    return dict(q=q, sw=sw, dw=dw, scores=sc, sel=sel, rowptr=rowptr, col=g_of, rq=rq, rs=rs,
                bn=bn, bk=bk)


def quant_act(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Activation INT4 per (token, 128-group), fp32 scale amax/7."""
    return mx.quantize_int4_g128(np.asarray(x, dtype=np.float32))


def weight_dense(prep: dict) -> tuple[np.ndarray, np.ndarray]:
    """(base weight, residual weight) as dense float64 matrices."""
    base = dequant_rows(prep["q"], prep["sw"])
    res = np.zeros_like(base)
    bn, bk = prep["bn"], prep["bk"]
    K = base.shape[1]
    for i, blk in enumerate(prep["sel"]):
        nb, g = blk // (K // bk), blk % (K // bk)
        res[nb * bn:(nb + 1) * bn, g * bk:(g + 1) * bk] = prep["rq"][i] * prep["rs"][i].astype(np.float64)[:, None]
    return base, res


def forward(x: np.ndarray, prep: dict) -> tuple[np.ndarray, np.ndarray]:
    """y in float64 and the tolerance scale sum |x_q| |w_q|.  The weight is the dense base plus
    the residual blocks (their sum is exact in float64: both are small integers times fp16
    scales), so y is one plain GEMM over it."""
    qx, sx = quant_act(x)
    xd = (qx.reshape(qx.shape[0], -1, 128) * sx.astype(np.float64)[..., None]).reshape(qx.shape)
    base, res = weight_dense(prep)
    w = base + res
    assert np.array_equal(w - base, res)                     # the sum above lost nothing
    return G.gemm_with_scale(xd, w)


def forward_grouped(x: np.ndarray, prep: dict) -> np.ndarray:
    """The same y computed literally as sum_g sx sw I_g (+ residual), with integer I_g (pin)."""
    qx, sx = quant_act(x)
    M, K = qx.shape
    N = prep["q"].shape[0]
    y = np.zeros((M, N))
    for g in range(K // 128):
        Ig = qx[:, g * 128:(g + 1) * 128] @ prep["q"][:, g * 128:(g + 1) * 128].T     # int64
        y += sx[:, g].astype(np.float64)[:, None] * prep["sw"][:, g].astype(np.float64)[None, :] * Ig
    bn = prep["bn"]
    for i, blk in enumerate(prep["sel"]):
        nb, g = blk // (K // 128), blk % (K // 128)
        Rg = qx[:, g * 128:(g + 1) * 128] @ prep["rq"][i].T                            # [M, 16]
        y[:, nb * bn:(nb + 1) * bn] += sx[:, g].astype(np.float64)[:, None] * \
            prep["rs"][i].astype(np.float64)[None, :] * Rg
    return y
