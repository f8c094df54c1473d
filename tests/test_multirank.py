"""Multi-rank host logic of the benchmark (replicas, weak scaling), on CPU with
two `gloo` ranks: the job time is the maximum over ranks and the throughput
counts every rank's work; ranks other than 0 leave the reference arm at once."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r's timed region took 10 + r ms, its end-to-end run 30 - r ms
        ms, e2e = bench.job_times(10.0 + rank, 30.0 - rank, world, "cpu")
        out[rank] = (ms, e2e, bench.job_throughput(2.0, 5, world, ms))
    finally:
        dist.destroy_process_group()


def test_job_time_is_max_over_ranks_and_throughput_counts_all_ranks():
    world = 2
    out = mp.get_context("spawn").Manager().dict()  # no fork of this multi-threaded process
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    for r in range(world):
        ms, e2e, value = out[r]
        assert ms == 11.0 and e2e == 30.0
        assert value == pytest.approx(2.0 * 5 * world / 0.011)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_times(4.0, 9.0, 1) == (4.0, 9.0)
    assert bench.job_throughput(1.5, 10, 1, 3.0) == pytest.approx(1.5 * 10 / 0.003)


def test_reference_arm_runs_on_rank_0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
