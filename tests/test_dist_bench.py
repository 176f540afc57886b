"""The multi-GPU bench path is N independent replicas: each rank times its own
copy of the workload and the job's time is the slowest rank's.  Checked here
with two gloo ranks on CPU (no GPU, no collective on the data path)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.reduce_max(times[rank], dist, "cpu")
        out[rank] = (m, bench.job_gbs(world, 1_000_000, 10, m))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [(3.0, 5.0), (7.5, 2.5)])
def test_replica_timing_takes_the_slowest_rank(times):
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, _free_port(), times, out), nprocs=world,
                           start_method="spawn")
        got = dict(out)
    worst = max(times)
    for r in range(world):
        m, gbs = got[r]
        assert m == worst
        assert gbs == pytest.approx(world * 1_000_000 * 10 / (worst * 1e-3) / 1e9)


def test_single_rank_needs_no_process_group():
    assert bench.reduce_max(4.0, None, "cpu") == 4.0
    assert bench.job_gbs(1, 2e9, 1, 1000.0) == pytest.approx(2.0)
