"""The multi-GPU (replica) path of bench.py on the CPU: two gloo ranks share
the slowest rank's time and report the whole job's bytes over it; the
reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 0.30 + 0.05 * rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(mine, "cpu")
        results[rank] = (ms, bench.whole_job_gbs(1_000_000_000, world, ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    manager = mp.Manager()
    results = manager.dict()
    mp.start_processes(_rank, args=(world, port, results), nprocs=world, join=True, start_method="spawn")
    assert set(results.keys()) == {0, 1}
    for r in range(world):
        ms, gbs = results[r]
        assert ms == pytest.approx(0.35)
        assert gbs == pytest.approx(2 * 1e9 / 0.35e-3 / 1e9)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
