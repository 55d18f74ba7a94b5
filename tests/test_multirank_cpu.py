"""The benchmark's multi-rank aggregation on CPU: two gloo ranks, each with
its own per-step time, agree on the slowest rank's time and on the
whole-job rate (weak scaling: every rank runs its own layer)."""

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


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    local_ms = [2.0, 3.0][rank]
    rate, ms = bench.whole_job_rate(75600, local_ms, world)
    bench.barrier(world)
    out[rank] = (rate, ms)
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_whole_job_rate():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn",
                           join=True)
        res = dict(out)
    for rank in range(world):
        rate, ms = res[rank]
        assert ms == 3.0
        assert rate == pytest.approx(2 * 75600 / 3e-3)


def test_single_rank_rate_needs_no_process_group():
    import bench
    rate, ms = bench.whole_job_rate(100, 4.0, 1)
    assert ms == 4.0 and rate == pytest.approx(100 / 4e-3)
