"""The bench's multi-rank plumbing on host-only ranks (gloo, world size 2):
the max-over-ranks timing reduction, and the reference arm under torchrun,
where rank 0 alone runs and prints one JSON line and rank 1 exits without
work. The GPU arm uses the same functions with NCCL."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench

    r, w, d = bench.dist_init()
    assert (r, w) == (rank, world) and d is not None and d.get_backend() == "gloo"
    v = bench.max_over_ranks(1.0 + 1.5 * rank, d)  # rank 0: 1.0, rank 1: 2.5
    bench.barrier(d)
    out[rank] = v
    dist.destroy_process_group()


@pytest.mark.skipif(torch.cuda.is_available(), reason="host-only ranks: with a GPU the ranks take NCCL")
def test_max_over_ranks_gloo():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_max_worker, args=(world, port, out), nprocs=world, start_method="spawn")
    assert dict(out) == {0: 2.5, 1: 2.5}


@pytest.mark.skipif(torch.cuda.is_available(), reason="host-only ranks: the GPU arm would take NCCL")
def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.2",
           "--config", "opt-1.3b"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 only
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
