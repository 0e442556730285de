"""The multi-rank (torchrun) host logic of bench.py on CPU with gloo,
world_size 2: every rank gets the max elapsed time over ranks, and the job
throughput counts the units of all ranks over that time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_ms = [120.0, 150.0][rank]
        m = bench.max_over_ranks(local_ms, world)
        thr = bench.job_throughput(1.0e12, world, 10, m)
        q.put((rank, m, thr))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, m, thr in res:
        assert m == 150.0
        assert thr == pytest.approx(2 * 1.0e12 * 10 / 0.150)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(42.0, 1) == 42.0
    assert bench.job_throughput(5.0, 1, 4, 2000.0) == pytest.approx(10.0)
