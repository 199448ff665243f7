"""Host logic of bench.py's multi-GPU run, on CPU: ranks are independent
replicas whose time is the slowest rank's (an all-reduce MAX over the
process group), and the whole-job value counts every rank's units.  Two
gloo ranks on 127.0.0.1 stand in for two GPUs.  The reference arm prints
from rank 0 only; the other ranks exit 0 without work."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        elapsed = [0.50, 0.75][rank]  # rank 1 is the slow one
        slowest = bench.max_over_ranks(elapsed, world, torch.device("cpu"))
        value = bench.replica_throughput(world, 1000, slowest)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "value": value}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank(tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    got = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(2)]
    for g in got:
        assert g["slowest"] == pytest.approx(0.75)
        assert g["value"] == pytest.approx(2 * 1000 / 0.75)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.25, 1, None) == 0.25
    assert bench.replica_throughput(1, 100, 0.5) == pytest.approx(200.0)


def test_reference_arm_prints_from_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
