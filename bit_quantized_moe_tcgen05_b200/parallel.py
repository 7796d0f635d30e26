"""N-sharded (column-parallel) quantized linear over several GPUs, one process per GPU.

The layer y = x W^T splits along N, the output features (rows of W): every rank holds a
contiguous run of N / world weight rows (a multiple of 128, whole 128-row weight tiles, and for VQ
weights whole 64-row QBlocks), runs its own slice of the product with the library's kernels on the
replicated activation, and the slices meet in one all-gather over the process group (NCCL over
NVLink / NVSwitch on GPUs).  No other exchange exists: the reduction over K stays inside each
rank's GEMM.  Expert-parallel MoE (token rows exchanged all-to-all before and after the experts)
is not built.
"""
from __future__ import annotations

import numpy as np


def shard_rows(N: int, world: int, rank: int, align: int = 128) -> tuple[int, int]:
    """Rows [n0, n1) of rank `rank` when N rows split over `world` ranks in runs of whole
    `align`-row tiles, as evenly as the tiles allow (earlier ranks take the extra tiles)."""
    if N % align != 0:
        raise ValueError(f"N = {N} is not a multiple of {align}")
    tiles = N // align
    if tiles < world:
        raise ValueError(f"{tiles} tiles of {align} rows cannot cover {world} ranks")
    base, extra = divmod(tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return t0 * align, t1 * align


def slice_weight(n0: int, n1: int, codes=None, scales=None, indices=None, codebooks=None,
                 qblock_n: int = 64) -> dict:
    """The host arrays of weight rows [n0, n1): codes / scales / indices by rows; packed VQ
    codebooks [N/64, K/64, ...] by QBlock rows (n0 and n1 multiples of 64)."""
    out = {}
    if codes is not None:
        out["codes"] = np.ascontiguousarray(codes[n0:n1])
    if scales is not None:
        out["scales"] = np.ascontiguousarray(scales[n0:n1])
    if indices is not None:
        out["indices"] = np.ascontiguousarray(indices[n0:n1])
    if codebooks is not None:
        assert n0 % qblock_n == 0 and n1 % qblock_n == 0
        out["codebooks"] = np.ascontiguousarray(codebooks[n0 // qblock_n:n1 // qblock_n])
    return out


def gather_columns(y_local, group=None):
    """[M, N] from every rank's [M, n_r] slice (rank order), by one all-gather: into one buffer
    with all_gather_into_tensor where the slices are equal (NCCL), else by a list all_gather of
    slices padded to the widest (collectives move equal-sized pieces), trimmed afterwards."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if world == 1:
        return y_local
    M, n = y_local.shape
    sizes = [torch.zeros(1, dtype=torch.int64, device=y_local.device) for _ in range(world)]
    dist.all_gather(sizes, torch.tensor([n], dtype=torch.int64, device=y_local.device), group=group)
    ns = [int(s.item()) for s in sizes]
    if len(set(ns)) == 1 and dist.get_backend(group) == "nccl":
        buf = torch.empty((world * M, n), dtype=y_local.dtype, device=y_local.device)
        dist.all_gather_into_tensor(buf, y_local.contiguous(), group=group)
        return buf.view(world, M, n).permute(1, 0, 2).reshape(M, world * n)
    w = max(ns)
    mine = torch.zeros((M, w), dtype=y_local.dtype, device=y_local.device)
    mine[:, :n] = y_local
    parts = [torch.empty((M, w), dtype=y_local.dtype, device=y_local.device) for _ in ns]
    dist.all_gather(parts, mine, group=group)
    return torch.cat([pt[:, :k] for pt, k in zip(parts, ns)], dim=1)


class ShardedQLinear:
    """A QLinear whose N rows are split over the ranks of `group`; forward returns the full
    [M, N] output on every rank.  Takes the same host arrays and keywords as QLinear (the full
    weight); each rank keeps only its slice on its own GPU."""

    def __init__(self, codes=None, scales=None, group=None, indices=None, codebooks=None,
                 **kw):
        import torch.distributed as dist
        from . import QLinear
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        N = (codes if codes is not None else indices).shape[0]
        self.N = N
        self.n0, self.n1 = shard_rows(N, self.world, self.rank)
        sl = slice_weight(self.n0, self.n1, codes=codes, scales=scales, indices=indices,
                          codebooks=codebooks)
        self.local = QLinear(sl.get("codes"), sl["scales"], indices=sl.get("indices"),
                             codebooks=sl.get("codebooks"), **kw)

    def forward(self, x, stream=None):
        y_local = self.local(x, stream=stream)
        return gather_columns(y_local, self.group)

    __call__ = forward

    def close(self) -> None:
        self.local.close()
