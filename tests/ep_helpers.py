"""Test infrastructure of the expert-parallel layer (mixture_experts_feed_b200.ep).

``OracleOps``: CPU stand-ins of the library entry points that
``ExpertParallelMoE`` calls, with the binding's signatures and contracts,
computed by the oracle in float64 and stored into the caller's tensors.  With
them the exchange logic runs on CPU ranks over gloo.

``LoopbackComm``: the exchanges of W ranks that run as threads of one
process on one GPU.  Every exchange is host-synchronised: each rank's stream
is synchronised before its tensors are posted and after its copies, and the
ranks meet at a barrier between posting and copying.  No kernel ever waits on
another rank's kernel.  For the peer-memory transport it also hands out the
other threads' buffer addresses (all on the one GPU) and a host barrier.
"""
from __future__ import annotations

import threading

import torch

import mixture_experts_feed_b200 as moe
import oracle


class OracleOps:
    Layer = moe.Layer

    @staticmethod
    def new_workspace(L, device=None, stream=None):
        return torch.zeros(1)

    @staticmethod
    def moe_route(L, x, w_router, corr_bias, tw, ti, sg, ws, stream=None):
        g = oracle.gate(x, w_router, corr_bias, L.E, L.k, L.S, L.route_scale, L.global_scale)
        tw.copy_(g["topk_w"])
        ti.copy_(g["topk_idx"])
        if sg is not None:
            sg.copy_(g["shared_gamma"])

    @staticmethod
    def moe_permute(L, ti, pm, x, off, ps, ip, xp, ws, stream=None):
        p = oracle.permute(ti.to(torch.int64), L.E, pm)
        R = int(p["offsets"][-1])
        off.copy_(p["offsets"])
        ps[:R].copy_(p["perm_slot"])
        ip.copy_(p["inv_perm"])
        if xp is not None:
            xp[:R].copy_(x[p["perm_slot"] // L.k])

    @staticmethod
    def moe_ep_dispatch_prep(L, off, ps, tw, row_w, counts, ws, stream=None):
        R = int(off[-1])
        row_w[:R].copy_(tw.reshape(-1)[ps[:R].to(torch.int64)])
        counts.copy_(off[1:] - off[:-1])

    @staticmethod
    def moe_expert_ffn(L, x, xp, off, ps, tw, sg, wgu, wd, wsgu, wsd, yr, ys, ws, stream=None):
        for e in range(L.E):
            a, b = int(off[e]), int(off[e + 1])
            if b == a:
                continue
            slots = torch.arange(a, b) if ps is None else ps[a:b].to(torch.int64)
            wts = tw.reshape(-1)[slots].double()
            yr[a:b].copy_(oracle.expert_mlp(xp[a:b].double(), wgu[e].double(), wd[e].double(), wts))
        for s in range(L.S):
            ys[s * L.T:(s + 1) * L.T].copy_(oracle.expert_mlp(x.double(), wsgu[s].double(),
                                                              wsd[s].double(), sg[:, s].double()))

    @staticmethod
    def moe_shared_ffn(L, x, sg, wsgu, wsd, ys, ws, stream=None):
        for s in range(L.S):
            ys[s * L.T:(s + 1) * L.T].copy_(oracle.expert_mlp(x.double(), wsgu[s].double(),
                                                              wsd[s].double(), sg[:, s].double()))

    @staticmethod
    def moe_combine(L, yr, ys, ip, out, ws, stream=None):
        acc = torch.zeros(L.T, L.H, dtype=torch.float64)
        for s in range(L.S):
            acc += ys[s * L.T:(s + 1) * L.T].double()
        ipv = ip.view(L.T, L.k).to(torch.int64)
        for j in range(L.k):
            live = ipv[:, j] >= 0
            acc[live] += yr[ipv[live, j]].double()
        out.copy_(acc)


class LoopbackComm:
    """Shared state of W thread ranks; ``bind(rank)`` gives a rank's comm."""

    def __init__(self, world: int):
        self.world = world
        self.barrier = threading.Barrier(world, timeout=120)
        self.box = {}

    def bind(self, rank: int) -> "_RankComm":
        return _RankComm(self, rank)


class _RankComm:
    def __init__(self, shared: LoopbackComm, rank: int):
        self.s, self.rank, self.world = shared, rank, shared.world

    def _sync(self):
        if torch.cuda.is_available():
            torch.cuda.current_stream().synchronize()

    def all_to_all_equal(self, out, inp):
        self._sync()
        self.s.box[("a2a", self.rank)] = inp
        self.s.barrier.wait()
        n = out.numel() // self.world
        for src in range(self.world):
            out[src * n:(src + 1) * n].copy_(self.s.box[("a2a", src)][self.rank * n:(self.rank + 1) * n])
        self._sync()
        self.s.barrier.wait()

    def exchange(self, sends, recvs):
        self._sync()
        mine = {}
        for peer, t in sends:
            mine.setdefault(peer, []).append(t)
        self.s.box[("p2p", self.rank)] = mine
        self.s.barrier.wait()
        taken = {}
        for peer, t in recvs:
            msgs = self.s.box[("p2p", peer)].get(self.rank, [])
            i = taken.get(peer, 0)
            src = msgs[i]
            if src.shape != t.shape:
                raise RuntimeError(f"rank {self.rank}: message {i} from {peer} has shape "
                                   f"{tuple(src.shape)}, expected {tuple(t.shape)}")
            t.copy_(src)
            taken[peer] = i + 1
        for peer, msgs in ((p, self.s.box[("p2p", p)].get(self.rank, [])) for p in range(self.world)):
            if taken.get(peer, 0) != len(msgs):
                raise RuntimeError(f"rank {self.rank}: {len(msgs) - taken.get(peer, 0)} "
                                   f"unreceived messages from {peer}")
        self._sync()
        self.s.barrier.wait()

    # the peer-memory transport: all ranks' buffers live on the one GPU, so a
    # rank's "peer" pointers are the other threads' tensors' addresses
    def all_gather(self, out, inp):
        self._sync()
        self.s.box[("ag", self.rank)] = inp
        self.s.barrier.wait()
        for src in range(self.world):
            out[src].copy_(self.s.box[("ag", src)])
        self._sync()
        self.s.barrier.wait()

    def device_barrier(self, device):
        self._sync()
        self.s.barrier.wait()

    def peer_pointers(self, tensors):
        self.s.box[("pp", self.rank)] = [t.data_ptr() for t in tensors]
        self.s.barrier.wait()
        out = [[self.s.box[("pp", src)][i] for src in range(self.world)] for i in range(len(tensors))]
        self.s.barrier.wait()
        return out


def rank_weights(inputs: dict, E: int, world: int, rank: int) -> dict:
    """The weights rank ``rank`` holds: its slice of the routed experts, the rest whole."""
    El = E // world
    w = {n: t for n, t in inputs.items() if n != "x"}
    w["w_gate_up"] = inputs["w_gate_up"][rank * El:(rank + 1) * El]
    w["w_down"] = inputs["w_down"][rank * El:(rank + 1) * El]
    return w
