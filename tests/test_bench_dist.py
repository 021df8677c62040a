"""The multi-rank plumbing of bench.py, run as two gloo ranks on the CPU: the barrier,
the max-over-ranks step time and the whole-job (weak-scaling) throughput."""

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


def _rank_main(rank: int, world: int, port: int, q):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    my_ms = 2.0 + rank  # rank 1 is the slow one
    ms = bench.max_over_ranks(my_ms, world)
    value = bench.job_throughput(1000.0, world, ms)
    bench.barrier(world)
    q.put((rank, ms, value))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_job_throughput(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, value in res:
        assert ms == 3.0  # the slowest rank's time, seen by every rank
        assert value == pytest.approx(1000.0 * world / 3e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.job_throughput(10.0, 1, 2.0) == pytest.approx(5000.0)
