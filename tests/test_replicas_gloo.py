"""The multi-process path of bench.py on CPU: two ranks over gloo.

The forward pass has no data-path exchange (every (b, h) slice is independent), so N GPUs run N
replicas of the workload; the job's time is the slowest rank's device time and its throughput
N times one replica's work over that time. These tests check that reduction and that arithmetic
with real processes, and that the reference arm does no work on ranks other than 0.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_main(rank, world, port, times, out_path):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        value, tok = bench.job_throughput(4.0e12, 1.0e6, ms, world)
        with open(f"{out_path}.{rank}", "w") as f:
            f.write(f"{ms} {value} {tok}\n")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput(tmp_path):
    import torch.multiprocessing as mp
    times = [3.0, 7.5]  # ms: rank 1 is the slower replica
    out = str(tmp_path / "res")
    mp.start_processes(_rank_main, args=(2, _free_port(), times, out), nprocs=2, join=True, start_method="spawn")
    for rank in range(2):
        ms, value, tok = (float(x) for x in open(f"{out}.{rank}").read().split())
        assert ms == 7.5  # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 4.0e12 / 7.5e-3 / 1e12)  # two replicas' work in that time
        assert tok == pytest.approx(2 * 1.0e6 / 7.5e-3)


def test_job_throughput_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    value, tok = bench.job_throughput(2.0e12, 5.0e5, 10.0, 1)
    assert value == pytest.approx(200.0) and tok == pytest.approx(5.0e7)


def test_reference_arm_other_ranks_do_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1", MASTER_PORT="29511")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
