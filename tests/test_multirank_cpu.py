"""The N > 1 path of bench.py on CPU: world-size-2 gloo process groups.

Each rank runs its own replica of the workload (the attention path shards by
(batch, head) with no exchange), so the only cross-rank steps are the
barrier and the max-over-ranks reduction of device timings, and the job
throughput counts every rank's units.  Those are exercised here with gloo,
through the same functions bench.py calls, together with its handling of
--gpus against the launcher's world size.
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
    # what torchrun sets for each rank; bench.py --gpus 2 reads it back
    env = {"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)}
    layout = bench.resolve_world(2, env)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = [3.0, 7.5][rank]           # per-rank step time of its replica
        slowest = bench.rank_step_time(my_ms, world)   # barrier, then max over ranks
        results[rank] = (layout, slowest, bench.job_throughput(1000, world, slowest))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_job_throughput():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()  # no fork of a multi-threaded process
    results = mgr.dict()
    mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
    for r in range(world):
        layout, slowest, thr = results[r]
        assert layout == (2, r, r)
        assert slowest == 7.5                            # every rank sees the slowest rank
        assert thr == pytest.approx(1000 * 2 / 7.5e-3)  # units of all ranks / slowest time


def test_gpus_argument_against_the_launcher():
    # a launcher with another world size: refused, not silently one rank
    with pytest.raises(SystemExit):
        bench.resolve_world(8, {"WORLD_SIZE": "1"})
    with pytest.raises(SystemExit):
        bench.resolve_world(0, {})
    assert bench.resolve_world(1, {}) == (1, 0, 0)
    # no launcher and N > 1: bench.py relaunches itself with one rank per GPU
    assert bench.resolve_world(4, {}) is None
    cmd = bench.launch_command(4, ["--gpus", "4", "--steps", "3"])
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert cmd[cmd.index("--nproc-per-node") + 1] == "4"
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]


def test_single_rank_is_identity():
    assert bench.max_over_ranks(4.25, 1) == 4.25
    assert bench.job_throughput(10, 1, 2.0) == pytest.approx(5000.0)
