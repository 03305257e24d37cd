"""The replicas-only multi-GPU plumbing of bench.py, on CPU with gloo (world size 2).

Each rank runs its own replica of the workload (no collective on the data path); the job time
is the slowest rank's, and the job throughput counts every rank's FLOPs.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    # rank r reports a different step time and kernel time
    got = bench.max_over_ranks([100.0 + 50.0 * rank, 7.0 - rank])
    value = bench.job_throughput(329.0e12, world, got[0] / 10)
    q.put((rank, got, value))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in out:
        assert got == [150.0, 7.0]                  # the slowest rank's time on every rank
        assert value == pytest.approx(2 * 329.0e12 / 15.0e-3 / 1e12)


def test_single_process_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.job_throughput(1e12, 1, 1000.0) == pytest.approx(1.0)
