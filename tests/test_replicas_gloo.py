"""Host logic of bench.py's replica mode on CPU, world size 2, gloo.

The layer has no exchange step, so N GPUs run N independent replicas; the
only cross-rank work is the timing reduction (max over ranks) and the
barriers around the timed region.  These run here as two CPU processes, and
``bench.py --gpus 2`` is run end to end (it starts its own two ranks under
torch.distributed.run) with the CPU reference arm.
"""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup(None)
    assert (w, r) == (world, rank)
    per_rank_ms = [3.0, 7.5][rank]
    bench.barrier(w)
    got = bench.max_over_ranks(per_rank_ms, w)
    q.put((rank, got))
    bench.finish(w)


def test_max_over_ranks_world2_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    results = dict(q.get(timeout=10) for _ in range(2))
    assert results == {0: 7.5, 1: 7.5}


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_bench_gpus2_starts_two_ranks_and_prints_one_line():
    """``bench.py --gpus 2`` with no outer launcher starts two ranks itself
    (the driver's plain call); rank 0 prints the one JSON line, n_gpus = 2,
    rank 1 prints nothing.  The CPU reference arm runs on the small fp32
    workload, so no GPU is needed."""
    import json
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--impl", "reference", "--workload", "tiny-f32-T64-H128-E8k2S1-I64",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["impl"] == "reference"
    assert line["value"] > 0
