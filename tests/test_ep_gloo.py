"""Expert parallelism, exchange logic on CPU: two gloo ranks, each with its
own tokens and half of the routed experts, run ExpertParallelMoE with the
oracle-backed stand-ins of the library ops (tests/ep_helpers.py).  Every
rank's output must equal the oracle's layer on its tokens, which checks the
count exchange, the host tables, and that every run of rows lands where the
expert GEMM expects it and comes back to its slot."""
from __future__ import annotations

import os
import socket
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, case, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path[:0] = [ROOT, TESTS]
    import datetime
    import torch.distributed as dist
    import moe_workloads as mw
    import oracle
    from ep_helpers import OracleOps, rank_weights
    from mixture_experts_feed_b200.ep import ExpertParallelMoE, TorchDistComm
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        T_rank, H, E, k, S, I, skew = case
        w = mw.tiny(T=T_rank * world, H=H, E=E, k=k, S=S, I=I, dtype="bf16", route_scale=2.5, seed=13)
        inputs = mw.generate(w, threads=1)
        if skew:                          # most tokens pick the first experts (one rank's)
            inputs["corr_bias"] = torch.linspace(0.6, -0.6, E)
        x = inputs["x"][rank * T_rank:(rank + 1) * T_rank].contiguous()
        pm = None
        if rank == 1:                     # padded tokens on one rank
            pm = (torch.arange(T_rank) % 5 == 2).to(torch.uint8)
        layer = ExpertParallelMoE(rank_weights(inputs, E, world, rank), E, k, S, w.route_scale,
                                  comm=TorchDistComm(), device="cpu", ops=OracleOps)
        out = layer(x, padding_mask=pm)
        ref = oracle.moe_forward({**inputs, "x": x}, E, k, S, w.route_scale, w.global_scale,
                                 padding_mask=pm)["out"]
        # rows kept in fp32, one rounding to bf16 at the end: within half a
        # bf16 ulp of the exact value, plus fp32 storage of the rows
        err = (out.double() - ref).abs()
        bound = ref.abs() * 2.0 ** -8 + 1e-6 * float(ref.pow(2).mean().sqrt())
        ok = bool((err <= bound).all())
        q.put((rank, ok, float(err.max()), layer.last_counts))
    finally:
        dist.destroy_process_group()


def _run(case, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    res = {}
    for _ in range(world):
        rank, ok, err, counts = q.get(timeout=10)
        res[rank] = (ok, err, counts)
    for rank, (ok, err, counts) in res.items():
        assert ok, f"rank {rank}: max|out - oracle| {err:.3e} over the bound"
    # every row sent is received somewhere: the send and receive totals agree
    sent = [sum(res[r][2][0]) for r in range(world)]
    got = [sum(res[r][2][1]) for r in range(world)]
    assert sum(sent) == sum(got)
    return res


def test_ep_world2_gloo_matches_oracle():
    _run((48, 128, 8, 3, 2, 64, False))


def test_ep_world2_gloo_skewed_load():
    """Most rows go to rank 0's experts; rank 1 receives few."""
    res = _run((40, 128, 8, 2, 1, 64, True))
    assert res[0][2][1][0] + res[0][2][1][1] > res[1][2][1][0] + res[1][2][1][1]


def test_ep_world4_gloo_matches_oracle():
    _run((20, 64, 8, 2, 1, 64, False), world=4)
