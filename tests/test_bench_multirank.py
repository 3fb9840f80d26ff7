"""The benchmark's multi-rank host logic on CPU: two gloo ranks, each timing its own replica. The
job's time is the slowest rank's and its throughput counts every rank's tokens (weak scaling)."""
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


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    local_seconds = 0.5 + rank          # rank 1 is the slow one
    t = bench.max_over_ranks(local_seconds, dist, torch.device("cpu"))
    value = bench.job_throughput(world, 4096, 10, t)
    q.put((rank, t, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, t, value in got:
        assert t == 1.5                                 # the slowest rank's time on every rank
        assert value == pytest.approx(2 * 4096 * 10 / 1.5)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(0.25, None, None) == 0.25
    assert bench.job_throughput(1, 4096, 100, 0.5) == 4096 * 100 / 0.5
