"""Host logic of bench.py's multi-process path, on CPU: the max over ranks of
the device time (the collective bench.py runs after its timed region, here over
gloo with two processes), the whole-job weak-scaling rate, and that ranks other
than 0 leave the reference arm without work or output."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, values, results):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        results[rank] = bench.max_over_ranks(values[rank], dist, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_processes():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        values = [12.5, 31.25]
        mp.start_processes(_rank_main, args=(2, _free_port(), values, results), nprocs=2, join=True,
                           start_method="spawn")
        assert results[0] == results[1] == 31.25


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, None, "cpu") == 7.0


def test_weak_scaling_rate_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 64 queries per rank per step, 4 ranks, 10 steps in 20 ms (slowest rank)
    assert bench.weak_scaling_rate(64, 4, 10, 20.0) == pytest.approx(64 * 4 * 10 / 0.02)


def test_reference_arm_on_other_ranks_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
