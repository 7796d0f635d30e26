"""MoE grouped FFN with CodeQuant-style cluster-codebook experts (oracle; test infrastructure only).

"CodeQuant: Unified Clustering and Quantization ...", abstract and Figure 1 (Stage 3-4): expert
weights are absorbed into cluster centroids and the deployed kernel decodes them through a lookup
table kept in SM shared memory (Figure 4).  Here each output row of an expert weight has 16 bf16
centroids and every weight is a 4-bit index into its row's centroids.  Activations are MXFP4
(E8M0-B32).  The FFN is the gated MLP of the PRQuant page's Eq. (1): h = act(g) * u with g, u the
gate and up projections; SiLU is the gate activation (the Qwen3-style models the pages use).

Readings: gate rows 0..I-1 and up rows I..2I-1 of the fused gate/up weight; the gate weights of a
token are the softmax over its top-k logits (top-k by value, ties to the lower expert id); the
token's output sums its k slot contributions in slot order.
"""
from __future__ import annotations

import numpy as np

from . import formats as F
from . import gemm as G
from . import hadamard as Hd
from . import mx


def route(logits: np.ndarray, k: int) -> dict:
    """Top-k routing.  Returns ids [T,k] (descending logit, ties to the lower id), gate weights
    [T,k] (softmax of the k selected logits, float64), counts [E], offsets [E+1] and the routed
    entries f = t*k + s listed expert by expert, ascending (t, s) inside an expert."""
    T, E = logits.shape
    order = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")
    ids = order[:, :k].astype(np.int64)
    sel = np.take_along_axis(logits.astype(np.float64), ids, axis=1)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    den = np.zeros((T, 1))
    for s in range(k):                                   # the k terms summed in slot order
        den[:, 0] += ex[:, s]
    gates = ex / den
    counts = np.bincount(ids.reshape(-1), minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    entries = np.argsort(ids.reshape(-1), kind="stable")
    return dict(ids=ids, gates=gates, counts=counts, offsets=offsets, entries=entries)


def cluster_weight(cent_bits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """W[r, j] = centroid[r, idx[r, j]] (float64); centroids given as bf16 bit patterns."""
    c = F.bf16_decode(cent_bits)
    return np.take_along_axis(c, idx.astype(np.int64), axis=1)


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g)) * u


def gate_up(xq: np.ndarray, r: dict, Wgu: list, I: int, k: int) -> tuple[np.ndarray, ...]:
    """Per routed entry (in expert-sorted order): g, u (float64), h = silu(g) * u, and the
    tolerance scales sum|x_q w| of g and u."""
    P = r["entries"].shape[0]
    g = np.empty((P, I))
    u = np.empty((P, I))
    tg = np.empty((P, I))
    tu = np.empty((P, I))
    for e in range(len(Wgu)):
        a, b = r["offsets"][e], r["offsets"][e + 1]
        if a == b:
            continue
        t = r["entries"][a:b] // k
        W = Wgu[e]
        y, ya = G.gemm_with_scale(xq[t], W)
        g[a:b], u[a:b] = y[:, :I], y[:, I:]
        tg[a:b], tu[a:b] = ya[:, :I], ya[:, I:]
    return g, u, swiglu(g, u), tg, tu


def down_combine(hq: np.ndarray, r: dict, Wd: list, T: int, k: int) -> tuple[np.ndarray, np.ndarray]:
    """out[t] = sum over slots s (in order) of gate[t,s] * W_d[e(t,s)] . h_q[t,s]; h_q is given in
    expert-sorted entry order.  Returns out [T, H] and its tolerance scale."""
    H = Wd[0].shape[0]
    ys = np.zeros((T * k, H))
    ts = np.zeros((T * k, H))
    for e in range(len(Wd)):
        a, b = r["offsets"][e], r["offsets"][e + 1]
        if a == b:
            continue
        f = r["entries"][a:b]
        ys[f], ts[f] = G.gemm_with_scale(hq[a:b], Wd[e])
    g = r["gates"].reshape(-1, 1)
    ys = (ys * g).reshape(T, k, H)
    ts = (ts * np.abs(g)).reshape(T, k, H)
    out = np.zeros((T, H))
    for s in range(k):
        out += ys[:, s]
    return out, ts.sum(axis=1)


def forward(xd: np.ndarray, logits: np.ndarray, Wgu: list, Wd: list, k: int,
            h_given: np.ndarray | None = None, had_x: bool = False, had_h: bool = False) -> dict:
    """The whole routed FFN.  xd: bf16 activations as float64 [T, H].  Wgu[e]: [2I, H] float64,
    Wd[e]: [H, I] float64.  h_given (optional): the intermediate h (expert-sorted order) to
    requantize instead of the oracle's own, for stage-wise comparison; it must then be float32
    values when had_h is set.  had_x / had_h: x, resp. h, passes the online block-32 Hadamard
    (hadamard.rotate_activation_f32) before its MXFP4 quantization; the weights given are then
    the rotated ones."""
    T = xd.shape[0]
    I = Wd[0].shape[1]
    xsrc = Hd.rotate_activation_f32(xd.astype(np.float32)).astype(np.float64) if had_x else xd
    xc, xs = mx.quantize_e8m0_b32(xsrc)
    xq = mx.dequant_e8m0_b32(xc, xs)
    r = route(logits, k)
    g, u, h, tg, tu = gate_up(xq, r, Wgu, I, k)
    hsrc = h if h_given is None else h_given
    if had_h:
        h32 = hsrc.astype(np.float32)
        assert h_given is None or np.array_equal(h32.astype(np.float64), hsrc), "h_given: float32 values"
        hsrc = Hd.rotate_activation_f32(h32).astype(np.float64)
    hc, hs = mx.quantize_e8m0_b32(hsrc)
    hq = mx.dequant_e8m0_b32(hc, hs)
    out, tout = down_combine(hq, r, Wd, T, k)
    return dict(route=r, g=g, u=u, h=h, tg=tg, tu=tu, h_codes=hc, h_scales=hs, out=out, t_out=tout,
                x_codes=xc, x_scales=xs)
