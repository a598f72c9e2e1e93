"""Expert parallelism of the Inkling MoE layer: the routed experts sharded
over W ranks, one GPU each (NeMo AutoModel Inkling ``layers`` page:
``GroupedExperts`` provides expert-parallel sharding, and the parallelizer
shards ``InklingMoE.experts`` over the expert-parallel mesh).

Partitioning.  Rank r owns the routed experts [r*El, (r+1)*El), El = E / W
(E a multiple of W), as slices ``w_gate_up [El, 2I, H]`` and
``w_down [El, H, I]``.  The router bank, the correction bias and the shared
experts are whole on every rank.  Every rank brings its own tokens.

One step on rank r (every arithmetic step is a kernel of the library; this
module holds the exchanges and their host-side bookkeeping only):

1. ``moe_route`` and ``moe_permute`` over its own T tokens.  The permuted
   rows are ordered by global expert, so the rows for rank d form one run
   ``[off[d*El], off[(d+1)*El])``, sub-ordered by expert.
2. ``moe_ep_dispatch_prep``: each permuted row's routing weight (it travels
   with the row) and the per-expert row counts.
3. Counts to every rank: an all-to-all of E int32 a rank.  Rank r then knows
   ``recv[s][e]``, the rows source s sends for its local expert e, and the
   host reads both count vectors (one device-to-host read a step).
4. Rows and weights to the experts' ranks: every (destination, expert) run
   of rows goes straight to its place in the destination's expert-major
   buffer (rows of local expert e from source 0, then source 1, ...), by
   grouped point-to-point sends and receives (NCCL between GPUs).  A rank's
   runs for itself are device-to-device copies.
5. ``moe_expert_ffn`` over the received rows: they are already grouped by
   local expert and in slot order (``perm_slot = None``), with their own
   weights.
6. The output rows go back the same way, into the sender's permuted order.
7. ``moe_shared_ffn`` over its own tokens and ``moe_combine``, as on one GPU.

Per rank and per step the exchange moves, for R_out rows sent and R_in rows
received: ``R_out*(H*dtype + 4)`` bytes out and ``R_in*(H*dtype + 4)`` in for
the rows and weights, and ``4*H`` bytes a row each way for the fp32 results
(``2*H`` with fp16 down projections, whose expert output rows are fp16).

The results equal the one-GPU layer's up to the order of rows inside the
expert GEMM tiles, which does not change any row's arithmetic.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import Layer, moe_combine, moe_ep_dispatch_prep, moe_expert_ffn, moe_permute, \
    moe_route, moe_shared_ffn, new_workspace


class TorchDistComm:
    """Exchanges over a ``torch.distributed`` process group (NCCL between
    GPUs; gloo between host processes).  Messages between one pair of ranks
    are matched in the order they are posted."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_to_all_equal(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        """Block s of ``inp`` (W equal blocks) to rank s; block s of ``out`` from rank s."""
        self.dist.all_to_all_single(out, inp, group=self.group)

    def exchange(self, sends: Sequence[Tuple[int, torch.Tensor]],
                 recvs: Sequence[Tuple[int, torch.Tensor]]) -> None:
        """Send each (peer, tensor) of ``sends`` and fill each (peer, tensor)
        of ``recvs``; to and from this rank itself the pairs are copied in
        order.  Returns when every receive has landed (in stream order)."""
        dist = self.dist
        own_out = [t for p, t in sends if p == self.rank]
        own_in = [t for p, t in recvs if p == self.rank]
        if len(own_out) != len(own_in):
            raise RuntimeError("unmatched messages to self")
        for src, dst in zip(own_out, own_in):
            dst.copy_(src)
        ops = [dist.P2POp(dist.isend, t, p, self.group) for p, t in sends if p != self.rank]
        ops += [dist.P2POp(dist.irecv, t, p, self.group) for p, t in recvs if p != self.rank]
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()


class _LibraryOps:
    """The library's entry points, as this module calls them."""
    Layer = Layer
    new_workspace = staticmethod(new_workspace)
    moe_route = staticmethod(moe_route)
    moe_permute = staticmethod(moe_permute)
    moe_ep_dispatch_prep = staticmethod(moe_ep_dispatch_prep)
    moe_expert_ffn = staticmethod(moe_expert_ffn)
    moe_shared_ffn = staticmethod(moe_shared_ffn)
    moe_combine = staticmethod(moe_combine)


def partition(E: int, world: int, rank: int) -> Tuple[int, int]:
    """The routed experts [first, first + El) that ``rank`` owns."""
    if world < 1 or E % world != 0:
        raise ValueError(f"{E} routed experts do not split evenly over {world} ranks")
    El = E // world
    return rank * El, El


class ExpertParallelMoE:
    """This rank's part of one Inkling MoE layer with its routed experts
    sharded over ``comm.world`` ranks.

    ``weights``: ``w_router [E+S, H]`` fp32, ``corr_bias [E]`` fp32,
    ``w_gate_up [El, 2I, H]`` and ``w_down [El, H, I]`` (this rank's
    experts, see ``partition``), ``ws_gate_up [S, 2I, H]``,
    ``ws_down [S, H, I]`` (all shared experts).  ``ops`` defaults to the
    library's kernels; a test may pass stand-ins with the same signatures.
    """

    def __init__(self, weights: dict, E: int, k: int, S: int, route_scale: float,
                 global_scale: float = 1.0, comm=None, device="cuda", ops=None):
        self.comm = comm if comm is not None else TorchDistComm()
        self.ops = ops if ops is not None else _LibraryOps
        self.W, self.rank = self.comm.world, self.comm.rank
        self.first, self.El = partition(E, self.W, self.rank)
        self.E, self.k, self.S = E, k, S
        self.device = device
        self.w = {n: t.to(device).contiguous() for n, t in weights.items()}
        if self.w["w_gate_up"].shape[0] != self.El or self.w["w_down"].shape[0] != self.El:
            raise ValueError(f"rank {self.rank} holds {self.El} routed experts")
        self.H = self.w["w_router"].shape[1]
        self.I = self.w["w_down"].shape[2]
        self.dtype = self.w["w_gate_up"].dtype
        self.down_f16 = self.w["w_down"].dtype == torch.float16   # fp16 down projections
        self.route_scale, self.global_scale = route_scale, global_scale
        self.last_counts = None       # (rows sent per destination, rows received per source)
        self._ws = []                 # the workspaces of the last call (status words)

    def layer(self, T: int) -> Layer:
        return self.ops.Layer(T, self.H, self.E, self.k, self.S, self.I, self.dtype,
                              self.route_scale, self.global_scale, self.down_f16)

    def __call__(self, x: torch.Tensor, padding_mask: Optional[torch.Tensor] = None) -> torch.Tensor:
        ops, dev, W, El, H = self.ops, self.device, self.W, self.El, self.H
        T = x.shape[0]
        L = self.layer(T)
        k, S, E = self.k, self.S, self.E
        ws = ops.new_workspace(L, device=dev)
        tw = torch.empty(T, k, dtype=torch.float32, device=dev)
        ti = torch.empty(T, k, dtype=torch.int32, device=dev)
        sg = torch.empty(T, S, dtype=torch.float32, device=dev) if S else None
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        ps = torch.empty(T * k, dtype=torch.int32, device=dev)
        ip = torch.empty(T * k, dtype=torch.int32, device=dev)
        xp = torch.empty(T * k, H, dtype=self.dtype, device=dev)
        row_w = torch.empty(T * k, dtype=torch.float32, device=dev)
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        pm = None if padding_mask is None else padding_mask.to(dev, torch.uint8).contiguous()
        w = self.w
        # 1-2: route and permute this rank's tokens; row weights and counts
        ops.moe_route(L, x, w["w_router"], w["corr_bias"], tw, ti, sg, ws)
        ops.moe_permute(L, ti, pm, x, off, ps, ip, xp, ws)
        ops.moe_ep_dispatch_prep(L, off, ps, tw, row_w, counts, ws)
        # 3: counts to every rank, then both count tables on the host
        recv_counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.comm.all_to_all_equal(recv_counts, counts)
        send = counts.view(W, El).cpu().tolist()          # [destination][local expert]
        recv = recv_counts.view(W, El).cpu().tolist()     # [source][local expert]
        send_start = _exclusive_scan([c for row in send for c in row])
        loc_tot = [sum(recv[s][e] for s in range(W)) for e in range(El)]
        loc_off = _exclusive_scan(loc_tot)
        R_in = loc_off[-1]
        dst_start = [[0] * El for _ in range(W)]          # [source][local expert]
        for e in range(El):
            run = loc_off[e]
            for s in range(W):
                dst_start[s][e] = run
                run += recv[s][e]
        self.last_counts = ([sum(r) for r in send], [sum(r) for r in recv])
        # 4: every (destination, expert) run of rows and weights to its place
        x_in = torch.empty(R_in, H, dtype=self.dtype, device=dev)
        w_in = torch.empty(R_in, dtype=torch.float32, device=dev)
        sends: List[Tuple[int, torch.Tensor]] = []
        recvs: List[Tuple[int, torch.Tensor]] = []
        for buf_out, buf_in in ((xp, x_in), (row_w, w_in)):
            for d in range(W):
                for e in range(El):
                    n, a = send[d][e], send_start[d * El + e]
                    if n:
                        sends.append((d, buf_out[a:a + n]))
            for s in range(W):
                for e in range(El):
                    n, b = recv[s][e], dst_start[s][e]
                    if n:
                        recvs.append((s, buf_in[b:b + n]))
        self.comm.exchange(sends, recvs)
        # 5: the local experts over the received rows (already grouped, in slot order)
        Ll = self.ops.Layer(R_in, H, El, 1, 0, self.I, self.dtype, self.route_scale,
                            self.global_scale, self.down_f16)
        y_dtype = torch.float16 if self.down_f16 else torch.float32   # the expert output rows
        y_in = torch.empty(R_in, H, dtype=y_dtype, device=dev)
        self._ws = [ws]
        if R_in > 0:
            off_loc = torch.tensor(loc_off, dtype=torch.int32).to(dev)
            ws_loc = ops.new_workspace(Ll, device=dev)
            self._ws.append(ws_loc)
            ops.moe_expert_ffn(Ll, x_in, x_in, off_loc, None, w_in, None, w["w_gate_up"],
                               w["w_down"], None, None, y_in, None, ws_loc)
        # 6: the output rows back into this rank's permuted order
        yr = torch.empty(T * k, H, dtype=y_dtype, device=dev)
        sends, recvs = [], []
        for s in range(W):
            for e in range(El):
                n, b = recv[s][e], dst_start[s][e]
                if n:
                    sends.append((s, y_in[b:b + n]))
        for d in range(W):
            for e in range(El):
                n, a = send[d][e], send_start[d * El + e]
                if n:
                    recvs.append((d, yr[a:a + n]))
        self.comm.exchange(sends, recvs)
        # 7: shared experts on this rank's tokens, then the fixed-order combine
        ys = None
        if S:
            ys = torch.empty(S * T, H, dtype=y_dtype, device=dev)
            ops.moe_shared_ffn(L, x, sg, w["ws_gate_up"], w["ws_down"], ys, ws)
        out = torch.empty(T, H, dtype=self.dtype, device=dev)
        ops.moe_combine(L, yr, ys, ip, out, ws)
        return out


def read_device_status(layer: "ExpertParallelMoE") -> int:
    """Read and clear the status words of the workspaces of the layer's last
    call (raises the binding's MoEError when a kernel recorded a problem)."""
    from . import read_device_status as _read
    code = 0
    for ws in layer._ws:
        code = code or _read(ws)
    return code


def _exclusive_scan(v: Sequence[int]) -> List[int]:
    out = [0]
    for c in v:
        out.append(out[-1] + c)
    return out
