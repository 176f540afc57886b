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
    with mp.get_context("spawn").Manager() as mgr:
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


def test_reference_arm_times_the_oracle_on_host_cores():
    # the reference arm needs no GPU: the oracle on every host core, one JSON line
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                          "tiny_decode", "--steps", "2", "--warmup", "1"], cwd=root,
                         capture_output=True, text=True, timeout=600, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["cores"] == (os.cpu_count() or 1)
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_cpu_baseline_reports_one_and_all_cores():
    import bench
    from verify_attention_paged_b200 import workloads as wl
    r = bench.cpu_baseline(wl.tiny_decode(), 0.4, threads=2)
    assert r["cores"] == 2 and r["kind"] == "oracle" and r["value"] > 0
    assert r["single_core"]["value"] > 0
