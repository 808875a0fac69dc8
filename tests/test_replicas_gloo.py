"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, the step time is the maximum over ranks
and the throughput counts the work of every rank (replicas, weak scaling).  No GPU involved."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = bench.max_over_ranks([1.0 + rank, 10.0 * (world - rank)], dist, "cpu")
        q.put((rank, times, bench.throughput(2e12, world, 4, times[0])))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, times, tops in out:
        assert times == [2.0, 20.0]
        # 2 ranks x 4 steps x 2e12 ops in 2 ms = 8000 TOPS
        assert tops == pytest.approx(2 * 4 * 2e12 / 2e-3 / 1e12)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks([3, 4]) == [3.0, 4.0]
