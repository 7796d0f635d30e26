"""PRQuant tail-block residual, as one augmented MXFP4 GEMM (oracle; test infrastructure only).

Follows "PRQuant: Permutation Residual Quantization for Low-Overhead Inference", §4 Method:
  * "Offline scaling and channel reordering": pick the top-k input channels of the down
    projection weight that are hardest to quantize and move them to contiguous tail blocks
    with a permutation P (Eq. 1: X W^T = (X P)(W P)^T).  The AWQ scaling D_alpha needs
    calibration activations and is taken as identity (alpha = 0).  "Hardest to quantize" is
    read as the largest per-column sum over output rows of the squared MXFP4 error.
  * "Offline residual augmentation": R_W = W~_tail - Q(W~_tail) (Eq. 2).  Eq. 3 is garbled on
    the page; it is read as Y^ = Q([Z~, Z~_tail]) Q([W~, R_W])^T, which the "Kernel design"
    paragraph spells out: W_aug = Q([W~, R_W]) prepared offline, the activation quantized once
    and the quantized tail appended with its block scales, and one GEMM over C + k.
"""
from __future__ import annotations

import numpy as np

from . import gemm as G
from . import mx


def _qw(search: bool):
    return mx.quantize_e8m0_b32_searched if search else mx.quantize_e8m0_b32


def column_errors(w: np.ndarray, search: bool = False) -> np.ndarray:
    """Per input channel: sum over output rows of (w - deq Q(w))^2, float64, accumulated in row
    order n = 0, 1, ... (a fixed order, so the top-k choice is reproducible to the last bit)."""
    codes, sb = _qw(search)(w)
    d = w - mx.dequant_e8m0_b32(codes, sb)
    acc = np.zeros(w.shape[1])
    for n in range(w.shape[0]):
        acc += d[n] * d[n]
    return acc


def select_tail(err: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest errors; ties go to the lower channel index; returned ascending."""
    order = sorted(range(err.shape[0]), key=lambda j: (-err[j], j))
    return np.array(sorted(order[:k]), dtype=np.int64)


def permutation(C: int, tail: np.ndarray) -> np.ndarray:
    """perm[j] = original channel at permuted position j: kept channels in ascending original
    order, then the tail channels in ascending original order."""
    mask = np.zeros(C, dtype=bool)
    mask[tail] = True
    return np.concatenate([np.nonzero(~mask)[0], np.asarray(tail, dtype=np.int64)])


def prepare(w: np.ndarray, k: int, search: bool = False) -> dict:
    """Offline preparation.  w float64 [N, C] (bf16 values), k % 32 == 0.  search = True quantizes
    every weight block with the E8M0-W block-scale search (§5.3) instead of the OCP rule.

    Returns perm [C], the augmented weight codes [N, C+k] (nibbles) and E8M0 bytes
    [N, (C+k)/32], and the residual R_W [N, k] for inspection.
    """
    N, C = w.shape
    assert C % 32 == 0 and k % 32 == 0 and 0 < k <= C
    q = _qw(search)
    tail = select_tail(column_errors(w, search), k)
    perm = permutation(C, tail)
    wp = w[:, perm]
    q_codes, q_sb = q(wp)
    r = wp[:, C - k:] - mx.dequant_e8m0_b32(q_codes[:, C - k:], q_sb[:, (C - k) // 32:])
    r_codes, r_sb = q(r)
    return dict(perm=perm, tail=tail,
                w_codes=np.concatenate([q_codes, r_codes], axis=1),
                w_sb=np.concatenate([q_sb, r_sb], axis=1),
                residual=r)


def quantize_activation_augmented(xp: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    """The augmented activation Q([X~, X~_tail]): quantize the permuted activation once, then
    append its quantized tail (codes and block scales) -- what both of PRQuant's tail
    constructions hand the GEMM (the online one by reading the tail twice, the offline one by
    writing the copy).  Returns codes [M, C+k], bytes [M, (C+k)/32]."""
    M, C = xp.shape
    codes, sb = mx.quantize_e8m0_b32(xp)
    return (np.concatenate([codes, codes[:, C - k:]], axis=1),
            np.concatenate([sb, sb[:, (C - k) // 32:]], axis=1))


def forward(xp: np.ndarray, prep: dict, k: int) -> tuple[np.ndarray, np.ndarray]:
    """y = Q([X~, X~_tail]) W_aug^T in float64; also the tolerance scale sum|x_q w_q|."""
    xc, xs = quantize_activation_augmented(xp, k)
    xd = mx.dequant_e8m0_b32(xc, xs)
    wd = mx.dequant_e8m0_b32(prep["w_codes"], prep["w_sb"])
    return G.gemm_with_scale(xd, wd)
