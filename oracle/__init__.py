"""CPU fp64 oracle of the Inkling MoE feed-forward forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / ``--impl reference`` legs use it.  It shares no code with the
CUDA path; the only module both read is ``moe_workloads`` (seeded inputs,
no layer arithmetic).

What it computes, step by step, from the NeMo AutoModel Inkling pages
(``layers`` page unless noted), in float64 with plain PyTorch CPU ops:

1. ``gate``: router logits over the whole gate weight bank (E routed rows then
   S shared rows), selection by sigmoid score plus correction bias, output
   weights from a softmax over the log-sigmoid of the selected routed logits
   concatenated with the shared logits, times route_scale * global_scale
   (``InklingGate`` docstring; ``InklingCorrectionBias.forward``).
2. ``swiglu_interleaved``: SwiGLU on the interleaved ``[g0, u0, g1, u1, ...]``
   last axis, scaled by the routing weight (``inkling_swiglu``).
3. ``expert_mlp``: one expert, fused gate/up projection, SwiGLU, down
   projection (``InklingSharedExperts``, ``inkling_swiglu``).
4. ``shared_experts``: the always-on experts, each weighted by its gamma and
   summed (``InklingSharedExperts`` docstring and ``forward``).
5. ``routed_experts``: every (token, choice) pair through its expert
   (``InklingMoE`` docstring: grouped routed experts).
6. ``moe_forward``: shared + routed, recombined per token
   (``InklingMoE.forward``).
7. ``permute``: the reference token order for grouped dispatch, rows ordered
   by (expert, token).
9. ``rmsnorm``: the feed-forward block's input norm (``InklingRMSNorm`` on
   the ``text`` page, the decoder layer's ``post_attention_layernorm``):
   ``x / sqrt(mean(x^2) + eps) * weight`` over the hidden axis, in float64,
   rounded once (round to nearest, ties to even) to the input's dtype.
8. ``dense_mlp``: the dense feed-forward layer (``InklingDenseMLP.forward``):
   fused interleaved gate/up projection, SwiGLU, down projection, times the
   layer's ``global_scale`` (the pages leave where it applies unstated; the
   output is scaled, which in exact arithmetic equals scaling h).

Readings taken where the pages are silent:
log-sigmoid applies to the whole concatenated vector, shared logits included;
the gammas are scaled like the routed weights; ties in the selection score go
to the lower expert index and the k chosen experts are returned in descending
score order; weights are stored ``[out, in]`` (the checkpoint form that needs
no more than a transposed view); the router has no norm; padded tokens take no routed
rows but still receive the shared experts; the dense layer's global_scale
multiplies its output.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(brute-force selection, closed-form weights, the sum invariant, the textbook
SwiGLU MLP special case, a library sort for the permutation, and a hand-worked
two-token example under ``tests/golden/``; for ``dense_mlp`` a textbook
SwiGLU MLP from separate gate and up matrices and a hand-worked closed-form
example).
"""
from __future__ import annotations

import os
from typing import Dict, Optional

import numpy as np
import torch
import torch.nn.functional as F

F64 = torch.float64


def _f64(t: torch.Tensor) -> torch.Tensor:
    """Exact widening of bf16 / fp32 CPU data to float64."""
    return t.detach().to("cpu").to(F64)


# ------------------------------------------------------------------ router
def router_logits(x: torch.Tensor, w_router: torch.Tensor) -> torch.Tensor:
    """z[t, e] = sum_h x[t, h] * Wr[e, h] for every row of the gate weight bank.

    ``InklingGate`` docstring: the gate weight bank additionally holds
    ``n_shared_experts`` rows; their logits join the normalisation.  The gate
    runs in fp32 on the pages (``gate_precision=torch.float32``); the oracle
    computes the exact value in float64.
    """
    return _f64(x) @ _f64(w_router).T


def selection_scores(z_routed: torch.Tensor, corr_bias: torch.Tensor) -> torch.Tensor:
    """sigmoid(z) + b on the routed logits only.

    ``InklingGate`` docstring (selection uses sigmoid scores plus a per-expert
    correction bias) and ``InklingCorrectionBias.forward`` (adds the bias to
    the routed scores).
    """
    return torch.sigmoid(z_routed) + _f64(corr_bias)[None, :]


def select_topk(scores: torch.Tensor, k: int) -> torch.Tensor:
    """Indices of the k best experts per token, best first.

    Order: score descending, then expert index ascending (ties go to the lower
    index).  A library stable lexicographic sort is the whole step.
    """
    s = scores.numpy()
    T, E = s.shape
    idx_grid = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((idx_grid, -s), axis=-1)   # primary key: -score; then index
    return torch.from_numpy(np.ascontiguousarray(order[:, :k])).to(torch.int64)


def routing_weights(z: torch.Tensor, idx: torch.Tensor, n_routed: int, n_shared: int,
                    route_scale: float, global_scale: float):
    """Weights of a given selection: p = softmax([logsig(z_sel_0..k-1) ++
    logsig(z_shared_0..S-1)]), every entry times route_scale * global_scale;
    the first k entries are the routed weights, the last S the shared gammas
    (``InklingGate`` docstring)."""
    E, S = n_routed, n_shared
    k = idx.shape[1]
    z_sel = torch.gather(z[:, :E], 1, idx)               # [T, k]
    v = torch.cat([F.logsigmoid(z_sel), F.logsigmoid(z[:, E:E + S])], dim=1)
    p = torch.softmax(v, dim=1)
    scale = float(route_scale) * float(global_scale)
    return p[:, :k] * scale, p[:, k:] * scale


def gate(x, w_router, corr_bias, n_routed: int, top_k: int, n_shared: int,
         route_scale: float, global_scale: float,
         given_topk_idx: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """``InklingGate.forward``: returns (topk_weights, topk_indices, shared_gammas).

    The correction bias enters the selection only; the weights follow
    ``routing_weights``.  ``given_topk_idx`` replaces the selection (used to
    evaluate the layer on a selection decided elsewhere, e.g. at a near-tie).
    """
    E, k, S = n_routed, top_k, n_shared
    z = router_logits(x, w_router)                       # [T, E+S]
    scores = selection_scores(z[:, :E], corr_bias)       # [T, E]
    idx = select_topk(scores, k) if given_topk_idx is None else given_topk_idx.to(torch.int64)
    topk_w, gamma = routing_weights(z, idx, E, S, route_scale, global_scale)
    # diagnostic: the selection margin between the k-th and (k+1)-th score
    ranked = torch.gather(scores, 1, select_topk(scores, min(k + 1, E)))
    gap = (ranked[:, k - 1] - ranked[:, k]) if k < E else torch.full((z.shape[0],), float("inf"), dtype=F64)
    return {"topk_w": topk_w, "topk_idx": idx, "shared_gamma": gamma,
            "logits": z, "scores": scores, "gap": gap}


# ------------------------------------------------------------------ experts
def swiglu_interleaved(G: torch.Tensor, routing_weights: torch.Tensor) -> torch.Tensor:
    """``inkling_swiglu``: last axis is [g0, u0, g1, u1, ...]; ``::2`` is gate,
    ``1::2`` is up; silu(g) * u is multiplied by the per-row routing
    weights (broadcast to ``[..., intermediate]``).  ``hidden_act='silu'``
    (``InklingTextConfig``): silu(g) = g * sigmoid(g).
    """
    g = G[..., 0::2]
    u = G[..., 1::2]
    return routing_weights * (g * torch.sigmoid(g)) * u


def expert_mlp(x_rows: torch.Tensor, w_gate_up: torch.Tensor, w_down: torch.Tensor,
               routing_weights: torch.Tensor) -> torch.Tensor:
    """One expert on a batch of rows: x @ Wgu^T -> interleaved SwiGLU (scaled)
    -> @ Wd^T.  Wgu is ``[2I, H]``, Wd is ``[H, I]`` (``[out, in]`` form)."""
    G = x_rows @ w_gate_up.T                             # [n, 2I]
    h = swiglu_interleaved(G, routing_weights[:, None])  # [n, I]
    return h @ w_down.T                                  # [n, H]


def shared_experts(x64: torch.Tensor, gamma: torch.Tensor, ws_gate_up, ws_down) -> torch.Tensor:
    """``InklingSharedExperts.forward(hidden_states, gammas)``: every token goes
    through every shared expert; expert s's output is weighted by gamma[:, s]
    before the sum."""
    out = torch.zeros_like(x64)
    for s in range(ws_gate_up.shape[0]):
        out += expert_mlp(x64, _f64(ws_gate_up[s]), _f64(ws_down[s]), gamma[:, s])
    return out


def routed_experts(x64: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
                   w_gate_up, w_down, padding_mask: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y[t, j] = expert_mlp of token t through expert topk_idx[t, j] with
    weight topk_w[t, j]; padded tokens get no routed rows (``InklingMoE.forward``:
    padded tokens never reach a routed expert).  Rows that chose
    the same expert are evaluated together; that grouping changes nothing but
    float64 rounding."""
    T, k = topk_idx.shape
    y = torch.zeros((T, k, x64.shape[1]), dtype=F64)
    live = torch.ones(T, dtype=torch.bool) if padding_mask is None else ~padding_mask.bool()
    for e in torch.unique(topk_idx[live]).tolist():
        t, j = torch.nonzero((topk_idx == e) & live[:, None], as_tuple=True)
        y[t, j] = expert_mlp(x64[t], _f64(w_gate_up[e]), _f64(w_down[e]), topk_w[t, j])
    return y


def moe_forward(inputs: Dict[str, torch.Tensor], n_routed: int, top_k: int, n_shared: int,
                route_scale: float, global_scale: float,
                tokens: Optional[torch.Tensor] = None,
                padding_mask: Optional[torch.Tensor] = None,
                threads: Optional[int] = None,
                given_topk_idx: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """``InklingMoE.forward``: out[t] = shared(t) + sum_j y[t, j], j ascending.

    ``tokens`` restricts the evaluation to a subset of token rows (the layer
    is per-token, so each row's result is the same as in a full run).
    ``given_topk_idx`` (rows matching ``tokens``) replaces the selection.
    Returns float64 tensors for the evaluated rows.
    """
    if threads is not None:
        torch.set_num_threads(threads)
    x = inputs["x"] if tokens is None else inputs["x"][tokens]
    pm = None
    if padding_mask is not None:
        pm = padding_mask if tokens is None else padding_mask[tokens]
    g = gate(x, inputs["w_router"], inputs["corr_bias"], n_routed, top_k, n_shared,
             route_scale, global_scale, given_topk_idx=given_topk_idx)
    x64 = _f64(x)
    sh = shared_experts(x64, g["shared_gamma"], inputs["ws_gate_up"], inputs["ws_down"])
    y = routed_experts(x64, g["topk_idx"], g["topk_w"], inputs["w_gate_up"], inputs["w_down"], pm)
    out = sh.clone()
    for j in range(top_k):
        out += y[:, j]
    return {"out": out, "shared": sh, "routed": y, **g}


def moe_forward_workload(inputs, w, tokens=None, padding_mask=None, threads=None,
                         given_topk_idx=None):
    """``moe_forward`` with the layer constants taken from a workload record."""
    return moe_forward(inputs, w.E, w.k, w.S, w.route_scale, w.global_scale,
                       tokens=tokens, padding_mask=padding_mask, threads=threads,
                       given_topk_idx=given_topk_idx)


# ------------------------------------------------------------- permutation
def permute(topk_idx: torch.Tensor, n_routed: int,
            padding_mask: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """Grouped-dispatch order: every live (token t, choice j) pair sorted by
    (expert, token) ascending (a library stable sort).

    Returns ``offsets[E+1]`` (exclusive scan of the per-expert counts),
    ``perm_slot[R]`` (for permuted row r, the slot t*k + j it came from) and
    ``inv_perm[T*k]`` (for slot t*k + j, its permuted row, -1 when padded).
    """
    idx = topk_idx.to(torch.int64).numpy()
    T, k = idx.shape
    live = np.ones(T, dtype=bool) if padding_mask is None else ~padding_mask.numpy().astype(bool)
    t_of = np.repeat(np.arange(T), k)
    e_of = idx.reshape(-1)
    keep = np.repeat(live, k)
    slots = np.nonzero(keep)[0]
    order = slots[np.lexsort((t_of[slots], e_of[slots]))]   # primary: expert, then token
    counts = np.bincount(e_of[slots], minlength=n_routed)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    inv = np.full(T * k, -1, dtype=np.int64)
    inv[order] = np.arange(order.size)
    return {"offsets": torch.from_numpy(offsets.astype(np.int64)),
            "perm_slot": torch.from_numpy(order.astype(np.int64)),
            "inv_perm": torch.from_numpy(inv),
            "counts": torch.from_numpy(counts.astype(np.int64))}


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


# ------------------------------------------------------------- dense layer
def dense_mlp(x: torch.Tensor, w_gate_up: torch.Tensor, w_down: torch.Tensor,
              global_scale: float = 1.0, tokens: Optional[torch.Tensor] = None) -> torch.Tensor:
    """``InklingDenseMLP.forward`` (``layers`` page): ``x`` of shape ``[..., H]``
    (any leading dims) through the fused interleaved projection ``w_gate_up``
    ``[2I, H]`` (row 2j gate_j, row 2j+1 up_j), SwiGLU (``inkling_swiglu`` with
    weight 1), the down projection ``w_down`` ``[H, I]``, times
    ``global_scale``.  Returns float64 of shape ``[..., H]``; with ``tokens``
    (indices into the flattened leading dims) only those rows, ``[n, H]``."""
    H = x.shape[-1]
    x64 = _f64(x).reshape(-1, H)
    if tokens is not None:
        x64 = x64[tokens]
    G = x64 @ _f64(w_gate_up).T
    h = swiglu_interleaved(G, torch.ones(G.shape[0], 1, dtype=F64))
    out = float(global_scale) * (h @ _f64(w_down).T)
    if tokens is not None:
        return out
    return out.reshape(*x.shape[:-1], H)


# ------------------------------------------------------------------ RMSNorm
def round_to_bf16(y: torch.Tensor) -> torch.Tensor:
    """Round float64 values once to the nearest bfloat16 (ties to even),
    returned as float64 holding bfloat16 values.  Normal range: keep the top
    7 fraction bits of the float64 pattern, rounding on the dropped 45 bits
    (adding 2^44 - 1 plus the kept last bit carries exactly when the dropped
    part is above half, or exactly half with an odd last bit).  Below 2^-126
    bfloat16 spacing is 2^-133: round y * 2^133 to an integer, ties to even.
    (A float64 -> float32 -> bfloat16 cast rounds twice and can differ.)"""
    a = y.detach().to("cpu", F64).numpy().copy()
    bits = a.view(np.uint64)
    lsb = (bits >> np.uint64(45)) & np.uint64(1)
    rb = ((bits + np.uint64((1 << 44) - 1) + lsb) >> np.uint64(45)) << np.uint64(45)
    r = rb.view(np.float64).copy()
    tiny = np.abs(a) < 2.0 ** -126
    r[tiny] = np.rint(a[tiny] * 2.0 ** 133) * 2.0 ** -133
    return torch.from_numpy(r)


def rmsnorm(x: torch.Tensor, weight: torch.Tensor, eps: float,
            out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    """``InklingRMSNorm.forward``: each row of the last axis divided by its
    root mean square (with ``eps`` added to the mean square), times the
    learned ``weight``; float64.  With ``out_dtype`` (the module returns the
    input's dtype) the float64 result is rounded once to it and returned in
    that dtype."""
    x64 = _f64(x)
    y = x64 / torch.sqrt((x64 * x64).mean(-1, keepdim=True) + float(eps)) * _f64(weight)
    if out_dtype is None:
        return y
    if out_dtype == torch.bfloat16:
        return round_to_bf16(y).reshape(y.shape).to(torch.float32).to(torch.bfloat16)
    if out_dtype == torch.float32:
        return torch.from_numpy(y.numpy().astype(np.float32))
    return y.to(out_dtype)
