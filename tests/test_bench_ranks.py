"""Host logic of the multi-rank bench (replicas only): max over ranks of the
timed region, whole-job throughput, and the CPU-oracle arm running on rank 0
only.  Runs as world-size-2 gloo ranks on the CPU."""
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        # the slowest rank's time is the job's time
        out[rank] = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_max_over_ranks_single():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5


def test_job_throughput_weak_scaling():
    # 32768 tokens per rank in 6 ms per step: N ranks process N replicas
    one = bench.job_throughput(32768, 1, 6.0)
    assert one == pytest.approx(32768 / 0.006)
    assert bench.job_throughput(32768, 4, 6.0) == pytest.approx(4 * one)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1", MASTER_PORT="29999")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
