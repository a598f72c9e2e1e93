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

Over peer memory (``transport="p2p"``: the GPUs of one node, NVLink) steps 2,
4 and 6 are kernels that store straight into other ranks' buffers.  Every
rank's permutation offsets (and token count) go to every rank in one
all-gather, from which each rank computes, on the host, where its rows land
in each owner's receive buffer and where each received run goes back.
``moe_ep_dispatch_p2p`` then reads each permuted row from x and stores it,
with its weight, into its owner's receive buffer (no x_perm copy, no
message); after a barrier over the ranks (an all-reduce on the stream) each
rank runs ``moe_expert_ffn`` on what it received, ``moe_ep_return_p2p``
stores each output row into its source's y rows, and after a second barrier
each rank combines as on one GPU.  The buffers other ranks store into
(``PeerBuffers``) are allocated once, with room for the largest step seen,
and their addresses exchanged once (CUDA IPC between processes); a step that
needs more room reallocates them on every rank, which all ranks decide alike
from the same counts.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import Layer, moe_combine, moe_ep_dispatch_p2p, moe_ep_dispatch_prep, moe_ep_return_p2p, \
    moe_expert_ffn, moe_permute, moe_route, moe_shared_ffn, new_workspace


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

    def all_gather(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        """Row s of ``out`` ([W, n]) is rank s's ``inp`` ([n])."""
        self.dist.all_gather_into_tensor(out.view(-1), inp, group=self.group)

    def device_barrier(self, device) -> None:
        """Every rank's work queued on its current stream before this call
        completes before any rank's work queued after it (an all-reduce on
        the stream: it cannot finish anywhere before every rank has entered
        it, and each rank enters it only after its earlier kernels)."""
        self.dist.all_reduce(torch.ones(1, device=device), group=self.group)

    def peer_pointers(self, tensors: Sequence[torch.Tensor]) -> List[List[int]]:
        """For each of ``tensors`` (the same list on every rank), the device
        address of every rank's tensor as mapped in this process: this rank's
        own, and the others' through CUDA IPC handles (GPUs of one node).  The
        mappings stay open as long as this object lives."""
        dist = self.dist
        mine = [(t.untyped_storage()._share_cuda_(), t.storage_offset() * t.element_size())
                for t in tensors]
        everyone = [None] * self.world
        dist.all_gather_object(everyone, mine, group=self.group)
        if not hasattr(self, "_mapped"):
            self._mapped = []
        out = []
        for i, t in enumerate(tensors):
            row = []
            for s in range(self.world):
                if s == self.rank:
                    row.append(t.data_ptr())
                    continue
                handle, offset = everyone[s][i]
                storage = torch.UntypedStorage._new_shared_cuda(*handle)
                self._mapped.append(storage)
                row.append(storage.data_ptr() + offset)
            out.append(row)
        return out


class _LibraryOps:
    """The library's entry points, as this module calls them."""
    Layer = Layer
    new_workspace = staticmethod(new_workspace)
    moe_route = staticmethod(moe_route)
    moe_permute = staticmethod(moe_permute)
    moe_ep_dispatch_prep = staticmethod(moe_ep_dispatch_prep)
    moe_ep_dispatch_p2p = staticmethod(moe_ep_dispatch_p2p)
    moe_ep_return_p2p = staticmethod(moe_ep_return_p2p)
    moe_expert_ffn = staticmethod(moe_expert_ffn)
    moe_shared_ffn = staticmethod(moe_shared_ffn)
    moe_combine = staticmethod(moe_combine)


class PeerBuffers:
    """The buffers of this rank that other ranks store into over peer memory
    (receive rows and weights for the dispatch, y rows for the return), all
    ranks' alike in size, and the tables of every rank's addresses as mapped
    in this process (int64 CUDA tensors of W pointers)."""

    def __init__(self, comm, H: int, dtype, y_dtype, recv_rows: int, back_rows: int, device):
        self.recv_rows, self.back_rows = recv_rows, back_rows
        self.x_in = torch.empty(max(recv_rows, 1), H, dtype=dtype, device=device)
        self.w_in = torch.empty(max(recv_rows, 1), dtype=torch.float32, device=device)
        self.y_back = torch.empty(max(back_rows, 1), H, dtype=y_dtype, device=device)
        px, pw, py = comm.peer_pointers([self.x_in, self.w_in, self.y_back])
        self.ptr_x = torch.tensor(px, dtype=torch.int64, device=device)
        self.ptr_w = torch.tensor(pw, dtype=torch.int64, device=device)
        self.ptr_y = torch.tensor(py, dtype=torch.int64, device=device)


def p2p_tables(offsets: Sequence[Sequence[int]], rank: int, El: int) -> dict:
    """Host-side placement of one step over peer memory, from every rank's
    permutation offsets ``offsets[s]`` (E + 1 ints, rows ordered by global
    expert).  Receiver d holds its rows by local expert el, then by source
    s: run (el, s) starts at loc[d][el] + sum over s' < s of rank s''s count
    of expert d*El + el.  Returns, for ``rank``: ``dst_base[e]`` (where its
    rows of expert e start in the owner's buffer), ``run_start`` (E + 1: the
    runs of what it receives, el-major), ``src_base[j]`` (run j's first row in
    its source's permuted order), ``loc`` (El + 1 offsets of its local
    experts), ``rows_in``, and ``max_rows_in`` over all ranks."""
    W = len(offsets)
    E = len(offsets[0]) - 1
    cnt = [[offsets[s][e + 1] - offsets[s][e] for e in range(E)] for s in range(W)]
    start = []            # start[d][s][el]
    loc_all = []
    for d in range(W):
        loc = [0]
        st = [[0] * El for _ in range(W)]
        for el in range(El):
            e = d * El + el
            run = loc[-1]
            for s in range(W):
                st[s][el] = run
                run += cnt[s][e]
            loc.append(run)
        start.append(st)
        loc_all.append(loc)
    dst_base = [start[e // El][rank][e % El] for e in range(E)]
    run_start, src_base = [], []
    for el in range(El):
        for s in range(W):
            run_start.append(start[rank][s][el])
            src_base.append(offsets[s][rank * El + el])
    run_start.append(loc_all[rank][El])
    return {"dst_base": dst_base, "run_start": run_start, "src_base": src_base,
            "loc": loc_all[rank], "rows_in": loc_all[rank][El],
            "max_rows_in": max(loc[El] for loc in loc_all)}


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
    ``transport``: ``"exchange"`` (grouped sends and receives through
    ``comm``) or ``"p2p"`` (stores into the other ranks' buffers over peer
    memory; ``comm`` then also provides ``all_gather``, ``device_barrier``
    and ``peer_pointers``).
    """

    def __init__(self, weights: dict, E: int, k: int, S: int, route_scale: float,
                 global_scale: float = 1.0, comm=None, device="cuda", ops=None,
                 transport: str = "exchange"):
        if transport not in ("exchange", "p2p"):
            raise ValueError(f"unknown transport {transport!r}")
        self.transport = transport
        self.peers = None             # PeerBuffers of the p2p transport, made on first use
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
        if self.transport == "p2p":
            return self._call_p2p(x, padding_mask)
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


    def _call_p2p(self, x: torch.Tensor, padding_mask: Optional[torch.Tensor]) -> torch.Tensor:
        ops, dev, W, El, H = self.ops, self.device, self.W, self.El, self.H
        T = x.shape[0]
        L = self.layer(T)
        k, S, E = self.k, self.S, self.E
        w = self.w
        ws = ops.new_workspace(L, device=dev)
        tw = torch.empty(T, k, dtype=torch.float32, device=dev)
        ti = torch.empty(T, k, dtype=torch.int32, device=dev)
        sg = torch.empty(T, S, dtype=torch.float32, device=dev) if S else None
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        ps = torch.empty(T * k, dtype=torch.int32, device=dev)
        ip = torch.empty(T * k, dtype=torch.int32, device=dev)
        pm = None if padding_mask is None else padding_mask.to(dev, torch.uint8).contiguous()
        # 1: route and permute (indices only: the dispatch reads the rows from x)
        ops.moe_route(L, x, w["w_router"], w["corr_bias"], tw, ti, sg, ws)
        ops.moe_permute(L, ti, pm, x, off, ps, ip, None, ws)
        # 2: every rank's offsets and token count, and the placement of this step
        mine = torch.cat([off, torch.tensor([T], dtype=torch.int32, device=dev)])
        every = torch.empty(W, E + 2, dtype=torch.int32, device=dev)
        self.comm.all_gather(every, mine)
        every = every.cpu().tolist()
        tab = p2p_tables([row[:E + 1] for row in every], self.rank, El)
        back_rows = max(row[E + 1] for row in every) * k
        recv_rows = tab["max_rows_in"]
        self.last_counts = ([every[self.rank][(d + 1) * El] - every[self.rank][d * El] for d in range(W)],
                            [every[s][(self.rank + 1) * El] - every[s][self.rank * El] for s in range(W)])
        y_dtype = torch.float16 if self.down_f16 else torch.float32
        p = self.peers
        if p is None or p.recv_rows < recv_rows or p.back_rows < back_rows:
            # every rank sees the same counts, so every rank reallocates here
            def grow(n, old):
                return max(n + n // 4, old)
            self.peers = p = PeerBuffers(self.comm, H, self.dtype, y_dtype,
                                         grow(recv_rows, p.recv_rows if p else 0),
                                         grow(back_rows, p.back_rows if p else 0), dev)
        dst_base = torch.tensor(tab["dst_base"], dtype=torch.int32).to(dev)
        run_start = torch.tensor(tab["run_start"], dtype=torch.int32).to(dev)
        src_base = torch.tensor(tab["src_base"], dtype=torch.int32).to(dev)
        # 3: rows and weights into their owners' receive buffers
        ops.moe_ep_dispatch_p2p(L, x, tw, ps, off, dst_base, W, p.ptr_x, p.ptr_w, p.recv_rows, ws)
        self.comm.device_barrier(dev)
        # 4: the local experts over what arrived (grouped by local expert, in slot order)
        R_in = tab["rows_in"]
        Ll = ops.Layer(R_in, H, El, 1, 0, self.I, self.dtype, self.route_scale, self.global_scale,
                       self.down_f16)
        y_in = torch.empty(max(R_in, 1), H, dtype=y_dtype, device=dev)
        self._ws = [ws]
        if R_in > 0:
            off_loc = torch.tensor(tab["loc"], dtype=torch.int32).to(dev)
            ws_loc = ops.new_workspace(Ll, device=dev)
            self._ws.append(ws_loc)
            ops.moe_expert_ffn(Ll, p.x_in[:R_in], p.x_in[:R_in], off_loc, None, p.w_in[:R_in], None,
                               w["w_gate_up"], w["w_down"], None, None, y_in[:R_in], None, ws_loc)
        # 5: the output rows back into their sources' permuted order
        ops.moe_ep_return_p2p(L, y_in, R_in, run_start, src_base, W, p.ptr_y, p.back_rows, ws)
        self.comm.device_barrier(dev)
        # 6: shared experts on this rank's tokens, then the fixed-order combine
        ys = None
        if S:
            ys = torch.empty(S * T, H, dtype=y_dtype, device=dev)
            ops.moe_shared_ffn(L, x, sg, w["ws_gate_up"], w["ws_down"], ys, ws)
        out = torch.empty(T, H, dtype=self.dtype, device=dev)
        ops.moe_combine(L, p.y_back[:T * k], ys, ip, out, ws)
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
