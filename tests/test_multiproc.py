"""The multi-GPU plumbing of bench.py on CPU: ranks as gloo processes (world size 2).
A prefill needs no collective (its (sequence, head) units are independent), so N GPUs run N
replicas; what the bench shares across ranks is the barrier and the max-over-ranks timing."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        out[rank] = bench.max_over_ranks(dist, torch, values[rank], torch.device("cpu"), world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    values = [3.25, 7.5]
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, values, out), nprocs=2, join=True)
        assert dict(out) == {0: 7.5, 1: 7.5}


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(None, torch, 4.0, torch.device("cpu"), 1) == 4.0


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    """bench.py --impl reference with 2 ranks: rank 0 times the CPU oracle and prints the one
    JSON line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
