"""The multi-rank side of bench.py on the CPU: world-size-2 gloo groups.

Each rank runs its own replica (the layer processes independent tokens), so
the only cross-rank steps are the timing reductions: the slowest rank's time
(max), the bytes every rank moved (sum), and the whole-job throughput built
from them.  The reference arm prints on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + rank           # rank 1 is the slow one
        nbytes = 1000.0 * (rank + 1)
        m = bench.over_ranks(ms, "max", "cpu")
        b = bench.over_ranks(nbytes, "sum", "cpu")
        v = bench.job_tokens_per_s(4, 100, world, m)
        out[rank] = (m, b, v)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_over_ranks_max_and_sum_world_2():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        m, b, v = out[r]
        assert m == 11.0                     # the slowest rank's time, on every rank
        assert b == 3000.0                   # every rank's bytes
        assert v == pytest.approx(4 * 100 * 2 / 0.011)   # all tokens over the slowest time


def test_single_process_is_the_identity():
    assert not dist.is_initialized()
    assert bench.over_ranks(7.5, "max", "cpu") == 7.5
    assert bench.over_ranks(7.5, "sum", "cpu") == 7.5
    assert bench.job_tokens_per_s(1, 1000, 1, 50.0) == pytest.approx(20000.0)


def test_reference_arm_prints_on_rank_0_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
