"""Seeded synthetic inputs for the Inkling MoE feed-forward layer.

This module is the one piece of code that both the CPU oracle (``oracle/``) and
the CUDA path (``mixture_experts_feed_b200``) consume.  It holds the workload
table and a seeded random generator, and nothing of the layer's arithmetic:
no routing, no activation, no matrix product.

Shapes follow the pages' statement of the layer (NeMo AutoModel Inkling
``layers`` page: ``InklingGate``, ``InklingSharedExperts``, ``inkling_swiglu``;
``configuration`` page: ``InklingTextConfig``).  Weight orientation is the
checkpoint's ``[out_features, in_features]`` form: the pages keep the fused
projection in the checkpoint's layout so that loading it takes no more than a
transposed view (``InklingSharedExperts`` docstring):

  x           [T, H]        activations, N(0, 1)
  w_router    [E+S, H] f32  gate weight bank: E routed rows then S shared rows,
                            N(0, 0.02^2) (``init_weights(init_std=0.02)``)
  corr_bias   [E]      f32  correction bias, U(-0.1, 0.1) or 0.5*log(Zipf)
  w_gate_up   [E, 2I, H]    fused projection, output rows interleaved
                            (row 2j = gate_j, row 2j+1 = up_j), N(0, 0.02^2)
  w_down      [E, H, I]     N(0, 0.02^2)
  ws_gate_up  [S, 2I, H]    shared experts, same law
  ws_down     [S, H, I]

Every tensor slice is drawn in fp32 from its own ``torch.Generator`` whose
seed is a fixed function of (workload seed, tensor id, slice index), then
rounded to nearest-even into the workload's dtype (the router tensors stay
fp32).  Because each expert slice has its own stream, any slice can be
regenerated alone and slices can be drawn in parallel threads with identical
results.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os
from typing import Dict, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "by_name", "generate", "slice_seed",
           "expert_slice", "zipf_bias", "flops", "tiny", "DenseWorkload",
           "DENSE_WORKLOADS", "dense_by_name", "generate_dense", "dense_flops"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One MoE-layer shape with its value distributions and seed."""

    name: str
    T: int            # tokens (leading dims flattened)
    H: int            # hidden size
    E: int            # routed experts
    k: int            # experts per token
    S: int            # shared experts
    I: int            # expert intermediate size
    dtype: str        # "f32" or "bf16" for x and the expert weights
    route_scale: float
    global_scale: float
    seed: int
    bias: str = "uniform"   # "uniform" U(-0.1,0.1) or "zipf" 0.5*log p_e, s=1.1
    init_std: float = 0.02

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The MoE workloads: a small fp32 layer, a mid-sized bf16 layer, three layers
# at InklingTextConfig's hidden size 6144 (prefill, one decode step, and a
# Zipf-skewed router), and the layer at InklingTextConfig's own MoE defaults.
WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("tiny-f32-T64-H128-E8k2S1-I64", 64, 128, 8, 2, 1, 64,
             "f32", 1.0, 1.0, seed=0),
    Workload("bf16-T4096-H2048-E64k6S2-I1024", 4096, 2048, 64, 6, 2, 1024,
             "bf16", 2.5, 1.0, seed=1),
    Workload("bf16-T8192-H6144-E128k8S1-I2048", 8192, 6144, 128, 8, 1, 2048,
             "bf16", 2.5, 1.0, seed=2),
    Workload("decode-bf16-T32-H6144-E128k8S1-I2048", 32, 6144, 128, 8, 1, 2048,
             "bf16", 2.5, 1.0, seed=3),
    Workload("zipf-bf16-T16384-H6144-E256k8S1-I1024", 16384, 6144, 256, 8, 1, 1024,
             "bf16", 2.5, 1.0, seed=4, bias="zipf"),
    # InklingTextConfig's own MoE defaults (hidden_size 6144, n_routed_experts
    # 256, num_experts_per_tok 6, n_shared_experts 2, moe_intermediate_size
    # 3072, route_scale 8.0) on a 4096-token batch: 29 GB of expert weights
    Workload("model-bf16-T4096-H6144-E256k6S2-I3072", 4096, 6144, 256, 6, 2, 3072,
             "bf16", 8.0, 1.0, seed=9),
]}

ORDERED = list(WORKLOADS.values())

# Layers sized for small ncu captures of the tcgen05 kernels (one kernel, a
# few launches, a few GB on the device): not parity workloads.  The same
# ad-hoc layer as tiny(T=2048, H=6144, E=24, k=3, S=1, I=2048, "bf16",
# route_scale=2.5, seed=3): the bench workload's H and I, 25 expert groups,
# about 1.9 GB of expert weights (more than L2).
PROFILE_WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("adhoc-T2048-H6144-E24k3S1-I2048-bf16", 2048, 6144, 24, 3, 1, 2048,
             "bf16", 2.5, 1.0, seed=3),
    # many tokens, small experts: x (201 MB) and the fp32 rows (805 MB) larger
    # than L2 for the HBM-bound kernels (norm, router, permutation, row
    # gather, combine), about 2 GB on the device in all
    Workload("adhoc-T16384-H6144-E16k2S1-I256-bf16", 16384, 6144, 16, 2, 1, 256,
             "bf16", 2.5, 1.0, seed=3),
    # one decode step over 17 expert groups (1.3 GB of weights, more than L2):
    # the weight-streaming expert GEMMs
    Workload("adhoc-decode-T32-H6144-E16k8S1-I2048-bf16", 32, 6144, 16, 8, 1, 2048,
             "bf16", 2.5, 1.0, seed=3),
    # the bench workload's routing (T=8192, E=128, k=8, S=1: the same top-k
    # and the same router K split) over a narrow layer, for the router kernels
    Workload("adhoc-T8192-H512-E128k8S1-I64-bf16", 8192, 512, 128, 8, 1, 64,
             "bf16", 2.5, 1.0, seed=3),
]}


def by_name(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    if name in PROFILE_WORKLOADS:
        return PROFILE_WORKLOADS[name]
    # allow 1-based position as a short name ("1".."6")
    if name.isdigit() and 1 <= int(name) <= len(ORDERED):
        return ORDERED[int(name) - 1]
    raise KeyError(f"unknown workload {name!r}; known: {list(WORKLOADS)}")


def tiny(T=16, H=64, E=6, k=2, S=1, I=32, dtype="f32", route_scale=1.0,
         global_scale=1.0, seed=11, bias="uniform") -> Workload:
    """A small ad-hoc workload for unit tests."""
    return Workload(f"adhoc-T{T}-H{H}-E{E}k{k}S{S}-I{I}-{dtype}", T, H, E, k, S, I,
                    dtype, route_scale, global_scale, seed, bias)


def flops(w: Workload, tokens: Optional[int] = None) -> Dict[str, float]:
    """Algorithmic flop counts (2 per multiply-add) on the real rows."""
    T = w.T if tokens is None else tokens
    routed = 6.0 * T * w.k * w.H * w.I
    shared = 6.0 * T * w.S * w.H * w.I
    router = 2.0 * T * w.H * (w.E + w.S)
    return {"routed": routed, "shared": shared, "router": router,
            "total": routed + shared + router}


# ---------------------------------------------------------------- generator
_TENSOR_IDS = {"x": 1, "w_router": 2, "corr_bias": 3, "w_gate_up": 4,
               "w_down": 5, "ws_gate_up": 6, "ws_down": 7,
               "dense_gate_up": 8, "dense_down": 9}


def slice_seed(seed: int, tensor: str, index: int = 0) -> int:
    """Seed of one tensor slice: a fixed integer mix of its three keys."""
    v = (seed * 1_000_003 + _TENSOR_IDS[tensor] * 7_919 + index * 104_729) & 0x7FFFFFFFFFFF
    return v ^ 0x5DEECE66D


def _normal(shape, std: float, seed: int) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def zipf_bias(E: int, s: float = 1.1) -> torch.Tensor:
    """0.5*log p_e with p_e proportional to (e+1)^-s (expert 0 most popular)."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    p = p / p.sum()
    return (0.5 * torch.log(p)).to(torch.float32)


def expert_slice(w: Workload, tensor: str, e: int) -> torch.Tensor:
    """One expert's slice of an expert weight tensor, in the workload dtype."""
    shapes = {"w_gate_up": (2 * w.I, w.H), "w_down": (w.H, w.I),
              "ws_gate_up": (2 * w.I, w.H), "ws_down": (w.H, w.I)}
    t = _normal(shapes[tensor], w.init_std, slice_seed(w.seed, tensor, e))
    return t.to(w.torch_dtype)


def _fill_experts(w: Workload, tensor: str, n: int, threads: int) -> torch.Tensor:
    shapes = {"w_gate_up": (2 * w.I, w.H), "w_down": (w.H, w.I),
              "ws_gate_up": (2 * w.I, w.H), "ws_down": (w.H, w.I)}
    out = torch.empty((n,) + shapes[tensor], dtype=w.torch_dtype)
    if n == 0:
        return out

    def one(e):
        src = _normal(shapes[tensor], w.init_std, slice_seed(w.seed, tensor, e))
        out[e].copy_(src)   # round-to-nearest-even into the workload dtype
        return e

    if threads <= 1:
        for e in range(n):
            one(e)
    else:
        with _cf.ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, range(n)))
    return out


def generate(w: Workload, pin_memory: bool = False, threads: Optional[int] = None,
             with_experts: bool = True) -> Dict[str, torch.Tensor]:
    """All inputs of one workload as CPU tensors (contiguous).

    ``x`` and the expert weights have the workload dtype; ``w_router`` and
    ``corr_bias`` are fp32.  ``pin_memory`` pins the large tensors for fast
    host->device copies.
    """
    if threads is None:
        threads = max(1, min(16, len(os.sched_getaffinity(0))))
    torch_threads = torch.get_num_threads()
    torch.set_num_threads(1 if threads > 1 else torch_threads)
    try:
        d: Dict[str, torch.Tensor] = {}
        d["x"] = _normal((w.T, w.H), 1.0, slice_seed(w.seed, "x")).to(w.torch_dtype)
        d["w_router"] = _normal((w.E + w.S, w.H), w.init_std, slice_seed(w.seed, "w_router"))
        if w.bias == "zipf":
            d["corr_bias"] = zipf_bias(w.E)
        else:
            g = torch.Generator(device="cpu")
            g.manual_seed(slice_seed(w.seed, "corr_bias"))
            d["corr_bias"] = (torch.rand((w.E,), generator=g, dtype=torch.float32) * 0.2 - 0.1)
        if with_experts:
            d["w_gate_up"] = _fill_experts(w, "w_gate_up", w.E, threads)
            d["w_down"] = _fill_experts(w, "w_down", w.E, threads)
            d["ws_gate_up"] = _fill_experts(w, "ws_gate_up", w.S, threads)
            d["ws_down"] = _fill_experts(w, "ws_down", w.S, threads)
    finally:
        torch.set_num_threads(torch_threads)
    if pin_memory:
        d = {k: v.pin_memory() for k, v in d.items()}
    return d


def token_sample(w: Workload, n: int, seed_offset: int = 0) -> torch.Tensor:
    """A fixed, sorted, seeded subset of token indices (for bounded oracle runs)."""
    n = min(n, w.T)
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed * 31 + 977 + seed_offset)
    return torch.randperm(w.T, generator=g)[:n].sort().values


def bf16_bytes(numel: int) -> int:
    return 2 * numel


def describe(w: Workload) -> str:
    return (f"T={w.T} H={w.H} E={w.E} k={w.k} S={w.S} I={w.I} {w.dtype} "
            f"route_scale={w.route_scale} global_scale={w.global_scale} seed={w.seed}"
            f" bias={w.bias}")


def weight_bytes(w: Workload) -> int:
    el = 4 if w.dtype == "f32" else 2
    return el * (w.E + w.S) * 3 * w.H * w.I + 4 * (w.E + w.S) * w.H + 4 * w.E



# ------------------------------------------------------------ dense layers
# The dense feed-forward layer of the model (``InklingDenseMLP`` on the
# ``layers`` page; ``dense_mlp_idx`` picks which decoder layer has it).  Its
# width is ``dense_intermediate_size`` when set, else ``intermediate_size``
# (24576 by default, ``InklingTextConfig``).  Weights in ``[out, in]`` form:
#
#   x          [T, H]    activations, N(0, 1)
#   gate_up    [2I, H]   fused projection, row 2j = gate_j, row 2j+1 = up_j,
#                        N(0, 0.02^2) (``InklingDenseMLP.init_weights``)
#   down       [H, I]    N(0, 0.02^2)
#
# The projections are drawn in slices of 256 rows, each from its own seed,
# so they can be drawn in parallel with identical results.

@dataclasses.dataclass(frozen=True)
class DenseWorkload:
    """One dense-MLP layer shape with its value distributions and seed."""

    name: str
    T: int
    H: int
    I: int
    dtype: str        # "f32" or "bf16"
    global_scale: float
    seed: int
    init_std: float = 0.02

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "DenseWorkload":
        return dataclasses.replace(self, **kw)


DENSE_WORKLOADS: Dict[str, DenseWorkload] = {w.name: w for w in [
    # the dense layer at the model's sizes (hidden 6144, intermediate 24576)
    DenseWorkload("dense-bf16-T8192-H6144-I24576", 8192, 6144, 24576, "bf16", 1.0, seed=5),
    # one decode step of the same layer: weight-streaming bound
    DenseWorkload("dense-decode-bf16-T32-H6144-I24576", 32, 6144, 24576, "bf16", 1.0, seed=6),
    # small cases the oracle finishes in seconds (ragged T, several tiles)
    DenseWorkload("dense-bf16-T300-H512-I640", 300, 512, 640, "bf16", 1.0, seed=7),
    DenseWorkload("dense-f32-T96-H128-I192", 96, 128, 192, "f32", 1.0, seed=8),
]}


def dense_by_name(name: str) -> DenseWorkload:
    if name in DENSE_WORKLOADS:
        return DENSE_WORKLOADS[name]
    raise KeyError(f"unknown dense workload {name!r}; known: {list(DENSE_WORKLOADS)}")


def dense_tiny(T=24, H=64, I=96, dtype="f32", global_scale=1.0, seed=21) -> DenseWorkload:
    """A small ad-hoc dense workload for unit tests."""
    return DenseWorkload(f"dense-adhoc-T{T}-H{H}-I{I}-{dtype}", T, H, I, dtype, global_scale, seed)


_DENSE_SLICE = 256


def _fill_rows(w: DenseWorkload, tensor: str, rows: int, cols: int, threads: int) -> torch.Tensor:
    out = torch.empty((rows, cols), dtype=w.torch_dtype)
    n = (rows + _DENSE_SLICE - 1) // _DENSE_SLICE

    def one(i):
        r0 = i * _DENSE_SLICE
        r1 = min(rows, r0 + _DENSE_SLICE)
        out[r0:r1].copy_(_normal((r1 - r0, cols), w.init_std, slice_seed(w.seed, tensor, i)))
        return i

    if threads <= 1:
        for i in range(n):
            one(i)
    else:
        with _cf.ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, range(n)))
    return out


def generate_dense(w: DenseWorkload, pin_memory: bool = False,
                   threads: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Inputs of one dense layer as CPU tensors: ``x``, ``w_gate_up``, ``w_down``."""
    if threads is None:
        threads = max(1, min(16, len(os.sched_getaffinity(0))))
    torch_threads = torch.get_num_threads()
    torch.set_num_threads(1 if threads > 1 else torch_threads)
    try:
        d = {"x": _normal((w.T, w.H), 1.0, slice_seed(w.seed, "x")).to(w.torch_dtype),
             "w_gate_up": _fill_rows(w, "dense_gate_up", 2 * w.I, w.H, threads),
             "w_down": _fill_rows(w, "dense_down", w.H, w.I, threads)}
    finally:
        torch.set_num_threads(torch_threads)
    if pin_memory:
        d = {k: v.pin_memory() for k, v in d.items()}
    return d


def dense_flops(w: DenseWorkload, tokens: Optional[int] = None) -> float:
    """Algorithmic flops of one dense layer (2 per multiply-add)."""
    T = w.T if tokens is None else tokens
    return 6.0 * T * w.H * w.I


def dense_token_sample(w: DenseWorkload, n: int, seed_offset: int = 0) -> torch.Tensor:
    """A fixed, sorted, seeded subset of token indices of a dense workload."""
    n = min(n, w.T)
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed * 31 + 977 + seed_offset)
    return torch.randperm(w.T, generator=g)[:n].sort().values


# ----------------------------------------------------------- norm weights
def norm_weight(H: int, seed: int, dtype: torch.dtype = torch.bfloat16,
                spread: float = 0.1) -> torch.Tensor:
    """A learned-looking RMSNorm scale: 1 + spread * N(0, 1) per channel (the
    module initialises it to ones; a spread keeps a missing weight visible)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 7919 + 17)
    return (1.0 + spread * torch.randn(H, generator=g, dtype=torch.float32)).to(dtype)


# rms_norm_eps of InklingTextConfig (1e-6), as the float32 the C ABI receives
RMS_NORM_EPS = float(torch.tensor(1e-6, dtype=torch.float32))
