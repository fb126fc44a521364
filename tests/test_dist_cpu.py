"""Multi-rank logic of the benchmark on CPU (gloo, world size 2): each rank runs its own
problem, timing is the max over ranks and throughput the sum; the oracle arm runs on
rank 0 only."""
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


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mx = bench.reduce_scalar(10.0 + rank, "max", world)
        sm = bench.reduce_scalar(1.5 * (rank + 1), "sum", world)
        out[rank] = (mx, sm)
    finally:
        dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:        # no fork of a multi-threaded process
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1] == (11.0, 4.5)


def test_reduce_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_scalar(3.25, "max", 1) == 3.25
    assert bench.reduce_scalar(3.25, "sum", 1) == 3.25


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_bench_rejects_mismatched_world():
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "1",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode != 0
