"""The N > 1 path of bench.py on CPU: world-size-2 gloo process groups.

Each rank runs its own replica of the workload (the attention path shards by
(batch, head) with no exchange), so the only cross-rank steps are the
barrier and the max-over-ranks reduction of device timings, and the job
throughput counts every rank's units.  Those are exercised here with gloo.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, results):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = [3.0, 7.5][rank]           # per-rank step time of its replica
        dist.barrier()
        slowest = bench.max_over_ranks(my_ms, world)
        results[rank] = (slowest, bench.job_throughput(1000, world, slowest))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_job_throughput():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
    for r in range(world):
        slowest, thr = results[r]
        assert slowest == 7.5                            # every rank sees the slowest rank
        assert thr == pytest.approx(1000 * 2 / 7.5e-3)  # units of all ranks / slowest time


def test_single_rank_is_identity():
    assert bench.max_over_ranks(4.25, 1) == 4.25
    assert bench.job_throughput(10, 1, 2.0) == pytest.approx(5000.0)
