"""Expert parallelism on one GPU: W ranks run as threads of this process, each
with its own tokens and its slice of the routed experts, exchanging through
LoopbackComm (host-synchronised copies: no kernel waits on another rank).
Every step of each rank runs in the library's kernels, as on W GPUs.

The ranks' outputs, concatenated, must equal bit for bit the one-GPU
moe_forward over all their tokens: each expert receives the same rows in the
same order (source rank by source rank is token order), and the router's K
split is the same at these sizes.  They are also held to the oracle's bar.
"""
from __future__ import annotations

import threading

import pytest
import torch

import moe_workloads as mw
import oracle
from ep_helpers import LoopbackComm, rank_weights
from moe_gpu_helpers import check_output, run_forward, to_device

pytestmark = pytest.mark.gpu


def run_ranks(inputs, world, T_rank, E, k, S, route_scale, pm=None, transport="exchange", calls=1):
    from mixture_experts_feed_b200.ep import ExpertParallelMoE, read_device_status
    shared = LoopbackComm(world)
    outs, counts, errs = [None] * world, [None] * world, []

    def run(r):
        try:
            torch.cuda.set_device(0)
            layer = ExpertParallelMoE(rank_weights(inputs, E, world, r), E, k, S, route_scale,
                                      comm=shared.bind(r), device="cuda", transport=transport)
            x = inputs["x"][r * T_rank:(r + 1) * T_rank].cuda()
            m = None if pm is None else pm[r * T_rank:(r + 1) * T_rank]
            o = layer(x, padding_mask=m)
            torch.cuda.synchronize()
            assert read_device_status(layer) == 0
            for _ in range(calls - 1):     # again, into the buffers of the first call
                again = layer(x, padding_mask=m)
                torch.cuda.synchronize()
                assert read_device_status(layer) == 0
                assert torch.equal(again, o)
            outs[r], counts[r] = o.cpu(), layer.last_counts
        except BaseException as e:    # noqa: BLE001 - reported below
            errs.append((r, e))
            shared.barrier.abort()

    th = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(300)
    assert not errs, errs
    return torch.cat(outs), counts


CASES = [
    # world, T a rank, H, E, k, S, I, skew, fp16 down projections
    (2, 256, 256, 16, 4, 1, 192, False, True),
    (2, 256, 256, 16, 4, 1, 192, False, False),
    (4, 128, 256, 16, 2, 2, 128, False, True),
    (4, 128, 128, 16, 2, 1, 64, True, True),    # every row to rank 0's experts: ranks 1-3 receive none
    (8, 64, 128, 16, 2, 1, 64, False, True),    # eight ranks of two experts each
]


@pytest.mark.parametrize("transport", ["exchange", "p2p"])
@pytest.mark.parametrize("case", CASES, ids=[f"W{c[0]}-T{c[1]}-H{c[2]}-E{c[3]}k{c[4]}S{c[5]}-I{c[6]}"
                                             + ("-skew" if c[7] else "") + ("-down-f16" if c[8] else "")
                                             for c in CASES])
def test_ep_virtual_ranks(case, transport):
    """``exchange``: rows and results travel as grouped sends and receives.
    ``p2p``: moe_ep_dispatch_p2p and moe_ep_return_p2p store them straight
    into the other ranks' buffers (here all on the one GPU), twice in a row
    into the same buffers."""
    world, T_rank, H, E, k, S, I, skew, down_f16 = case
    w = mw.tiny(T=T_rank * world, H=H, E=E, k=k, S=S, I=I, dtype="bf16", route_scale=2.5, seed=23)
    inputs = mw.generate(w, threads=4)
    if skew:
        inputs["corr_bias"] = torch.zeros(E)
        inputs["corr_bias"][:E // world] = 3.0
    pm = (torch.arange(w.T) % 7 == 4).to(torch.uint8)
    rank_inputs = dict(inputs)
    if down_f16:   # the ranks hold the exact fp16 copies of the down weights
        rank_inputs["w_down"] = inputs["w_down"].to(torch.float16)
        rank_inputs["ws_down"] = inputs["ws_down"].to(torch.float16)
    out_ep, counts = run_ranks(rank_inputs, world, T_rank, E, k, S, w.route_scale, pm=pm,
                               transport=transport, calls=2 if transport == "p2p" else 1)
    if skew:
        assert all(sum(counts[r][1]) == 0 for r in range(1, world))
    L = __import__("mixture_experts_feed_b200").Layer.from_workload(w, down_f16=down_f16)
    one = run_forward(L, to_device(inputs, down_f16=down_f16), padding_mask=pm)
    assert torch.equal(out_ep, one["out"]), "expert-parallel output differs from the one-GPU layer"
    ref = oracle.moe_forward_workload(inputs, w, padding_mask=pm,
                                      given_topk_idx=one["topk_idx"].to(torch.int64))
    rel = check_output(out_ep, ref["out"], torch.bfloat16, "expert-parallel out", strict=False)
    print(f"W={world} {transport}: rows sent {[sum(c[0]) for c in counts]}, received "
          f"{[sum(c[1]) for c in counts]}; max|out - oracle|/RMS = {rel:.4f}")
