"""The N-sharded (column-parallel) linear's host logic on CPU: row ranges, weight slicing and the
all-gather of output slices, over gloo with world size 2 (one process per rank).  The per-rank
product stands in for the rank's GPU GEMM; the GPU path itself runs on one GPU here."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_quantized_moe_tcgen05_b200 import parallel as P


def test_shard_rows_cover_all_tiles():
    for N, world in [(2560, 2), (2560, 8), (1280, 3), (128 * 7, 7), (8192, 8)]:
        got = [P.shard_rows(N, world, r) for r in range(world)]
        assert got[0][0] == 0 and got[-1][1] == N
        for (a0, a1), (b0, b1) in zip(got, got[1:]):
            assert a1 == b0
        sizes = [b - a for a, b in got]
        assert all(s % 128 == 0 and s > 0 for s in sizes)
        assert max(sizes) - min(sizes) <= 128          # as even as whole tiles allow
    with pytest.raises(ValueError):
        P.shard_rows(128, 2, 0)                        # one tile cannot cover two ranks
    with pytest.raises(ValueError):
        P.shard_rows(100, 1, 0)


def test_slice_weight_vq_codebooks_follow_qblocks():
    N, K = 512, 256
    idx = np.arange(N * K // 4, dtype=np.int64).reshape(N, K // 4) % 251
    cb = np.arange(N // 64 * K // 64 * 4, dtype=np.int64).reshape(N // 64, K // 64, 4)
    sb = np.arange(N * K // 16).reshape(N, K // 16) % 200
    sl = P.slice_weight(128, 384, scales=sb, indices=idx, codebooks=cb)
    assert np.array_equal(sl["indices"], idx[128:384])
    assert np.array_equal(sl["scales"], sb[128:384])
    assert np.array_equal(sl["codebooks"], cb[2:6])


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, N: int, q) -> None:
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        g = np.random.default_rng(0)                   # every rank draws the same full operands
        M, K = 5, 64
        W = torch.from_numpy(g.standard_normal((N, K)))
        x = torch.from_numpy(g.standard_normal((M, K)))
        n0, n1 = P.shard_rows(N, world, rank)
        y_local = x @ W[n0:n1].T                       # the rank's slice of the product
        y = P.gather_columns(y_local)
        q.put((rank, torch.equal(y, x @ W.T), tuple(y.shape)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N", [512, 640])             # 640: uneven slices (3 + 2 tiles)
def test_gather_columns_world2(N):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, N, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, same, shape in results:
        assert same, rank
        assert shape == (5, N)
