"""The N > 1 host path of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank of `bench.py --gpus N` runs an independent stream (replicas, weak
scaling); the only cross-rank steps are the barrier and the max over ranks of
the elapsed time, and the job's value is every rank's frames over that time.
These tests run those steps with the gloo backend, and check that under a
multi-rank launch only rank 0 runs and prints the reference arm.
"""
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as tdist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, elapsed, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        tdist.barrier()
        seconds = bench.max_over_ranks(elapsed[rank], "cpu")
        value = bench.job_throughput(3, 10, world, seconds)
        out[rank] = (seconds, value)
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_rank_and_the_job_value():
    world, port = 2, _free_port()
    elapsed = [0.25, 0.4]                 # rank 1 is the slow one
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, elapsed, out), nprocs=world, join=True)
    assert out[0] == out[1]               # every rank computes the same job figure
    seconds, value = out[0]
    assert seconds == 0.4
    assert value == pytest.approx(3 * 10 * 2 / 0.4)   # all ranks' frames over the slowest rank's time


def test_max_over_ranks_is_identity_without_a_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not tdist.is_initialized()
    assert bench.max_over_ranks(1.5, "cpu") == 1.5


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""         # rank 1 exits without work or output
