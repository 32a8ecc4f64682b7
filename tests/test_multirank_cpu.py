"""The multi-rank bench path on CPU: two gloo ranks (no GPU).

The encoder partitions into independent problems, so ranks exchange nothing on the data path; the
only collective is the max over ranks of the timed region, which is what is tested here.
"""

from __future__ import annotations

import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(values[rank], dist)
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    world = 2
    values = [3.5, 7.25]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), values, out), nprocs=world, join=True)
        assert dict(out) == {0: 7.25, 1: 7.25}


def test_weak_scaling_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.weak_scaling_value(1_000_000, 1, 1.0) == pytest.approx(1000.0)
    assert bench.weak_scaling_value(1_000_000, 4, 2.0) == pytest.approx(2000.0)
    assert bench.max_over_ranks(5.0) == 5.0


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
