"""The multi-process side of bench.py on CPU: world size 2 over gloo.  Each rank times its own
replica; the reported time is the slowest rank's and the value counts every rank's units over that
time.  Ranks other than 0 of the reference arm print nothing and exit 0."""

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


def _rank(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        slow = bench.slowest_rank_ms(ms, world)
        out[rank] = (slow, bench.whole_job_rate(1000.0, 4, world, slow))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        slow, rate = out[r]
        assert slow == 15.0
        assert rate == world * 1000.0 * 4 / 15e-3


def test_single_process_is_unchanged():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.slowest_rank_ms(7.5, 1) == 7.5
    assert bench.whole_job_rate(10.0, 2, 1, 4.0) == 10.0 * 2 / 4e-3


@pytest.mark.parametrize("config", ["prefill", "decode", "sweep", "dense_decode", "shared_prefill"])
def test_reference_arm_on_a_non_zero_rank_prints_nothing(config):
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", config, "--steps", "1", "--warmup", "0"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""
