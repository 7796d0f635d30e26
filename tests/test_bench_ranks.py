"""The multi-rank host logic of bench.py on CPU: world size 2 over gloo, one process per rank.
Each rank reports its own device times; every rank must see the element-wise maximum (the
slowest rank), and the whole-job throughput is the ranks' summed work over that time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    import datetime
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        mine = [1.0 + rank, 5.0 - rank]                  # rank 0: [1, 5], rank 1: [2, 4]
        got = bench.max_over_ranks(mine, torch.device("cpu"))
        thr = bench.job_throughput(0.5, world, got[0])
        q.put((rank, got, thr))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, thr in results:
        assert got == [2.0, 5.0], (rank, got)
        # 2 ranks x 0.5 units per step over 2 ms = 500 units / s
        assert thr == pytest.approx(2 * 0.5 / 2e-3)


def test_single_process_without_group_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.5], torch.device("cpu")) == [3.0, 4.5]
    assert bench.job_throughput(2.0, 1, 4.0) == pytest.approx(500.0)
