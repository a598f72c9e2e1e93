"""GPU parity of the feed-forward block's RMSNorm (moe_rmsnorm) and of the
pre-norm entry points (moe_forward_prenorm, moe_dense_mlp_prenorm) against the
CPU fp64 oracle.

The norm is bit-exact: both sides compute it in fp64 and round once (to
nearest, ties to even) into the input dtype.  Downstream the oracle runs the
layer on its own normalised input, so the selection, weight and output bars
of the MoE and dense parity tests apply unchanged.
"""
from __future__ import annotations

import pytest
import torch

import moe_workloads as mw
import oracle
from moe_gpu_helpers import check_output, run_chain, to_device
from test_gpu_parity import check_all

pytestmark = pytest.mark.gpu

try:
    import mixture_experts_feed_b200 as moe
except ImportError:   # collected on CPU-only machines too; the gpu marker deselects
    moe = None

EPS = mw.RMS_NORM_EPS


def gpu_rmsnorm(x, w, eps=EPS, inplace=False):
    xd = x.cuda().contiguous()
    out = xd if inplace else torch.empty_like(xd)
    moe.moe_rmsnorm(xd, w.cuda(), out, eps)
    torch.cuda.synchronize()
    return out.cpu()


@pytest.mark.parametrize("T,H,dtype", [(300, 512, torch.bfloat16), (1, 64, torch.bfloat16),
                                       (8192, 6144, torch.bfloat16), (77, 192, torch.float32),
                                       (1000, 2048, torch.float32),
                                       (1001, 8192, torch.bfloat16),    # 1024 vectors: 4 a thread
                                       (33, 8256, torch.bfloat16),      # longer rows: streamed kernel
                                       (20, 4160, torch.float32),       # streamed, fp32
                                       (5, 2112, torch.bfloat16)])      # 264 vectors, ragged team
def test_rmsnorm_bitexact(T, H, dtype):
    g = torch.Generator().manual_seed(T + H)
    x = torch.randn(T, H, generator=g).to(dtype)
    x[0, : H // 2] *= 1e-3                      # a row with a small scale
    w = mw.norm_weight(H, seed=T, dtype=dtype)
    got = gpu_rmsnorm(x, w)
    want = oracle.rmsnorm(x, w, EPS, out_dtype=dtype)
    assert got.dtype == dtype
    bad = (got != want).sum().item()
    assert bad == 0, f"{bad} of {got.numel()} elements differ from the single rounding"


def test_rmsnorm_in_place_and_zero_row():
    x = torch.randn(64, 256).to(torch.bfloat16)
    x[5] = 0                                     # mean square 0: sqrt(eps) only
    w = mw.norm_weight(256, seed=1)
    want = oracle.rmsnorm(x, w, EPS, out_dtype=torch.bfloat16)
    assert torch.equal(gpu_rmsnorm(x, w, inplace=True), want)
    assert torch.equal(want[5], torch.zeros(256, dtype=torch.bfloat16))


def run_prenorm(w, inputs, nw, down_f16=False):
    L = moe.Layer.from_workload(w, down_f16=down_f16)
    d = to_device(inputs, down_f16=down_f16)
    ws = moe.new_workspace(L)
    T, k, S, H = w.T, w.k, w.S, w.H
    out = torch.empty(T, H, dtype=w.torch_dtype, device="cuda")
    tw = torch.empty(T, k, device="cuda")
    ti = torch.empty(T, k, dtype=torch.int32, device="cuda")
    sg = torch.empty(T, S, device="cuda") if S else None
    moe.moe_forward_prenorm(L, d["x"], nw.cuda(), EPS, d["w_router"], d["corr_bias"],
                            d["w_gate_up"], d["w_down"], d.get("ws_gate_up") if S else None,
                            d.get("ws_down") if S else None, out, ws, topk_w=tw, topk_idx=ti,
                            shared_gamma=sg)
    torch.cuda.synchronize()
    moe.read_device_status(ws)
    r = {"out": out.cpu(), "topk_idx": ti.cpu(), "topk_w": tw.cpu(),
         "shared_gamma": sg.cpu() if S else None}
    return r, d, L


@pytest.mark.parametrize("shape", [(300, 256, 12, 3, 2, 320, "bf16"), (77, 192, 10, 2, 3, 192, "f32")],
                         ids=["bf16-T300", "f32-T77"])
def test_forward_prenorm_small(shape):
    T, H, E, k, S, I, dtype = shape
    w = mw.tiny(T=T, H=H, E=E, k=k, S=S, I=I, dtype=dtype, route_scale=2.5, seed=9)
    inputs = mw.generate(w, threads=4)
    nw = mw.norm_weight(H, seed=3, dtype=w.torch_dtype)
    r, d, L = run_prenorm(w, inputs, nw)
    # the oracle's own normalised input, then the layer's parity bars
    xn = oracle.rmsnorm(inputs["x"], nw, EPS, out_dtype=w.torch_dtype)
    check_all(w, {**inputs, "x": xn}, r)
    # the same kernels as the op chain on the normalised input: bitwise equal
    xn_gpu = torch.empty_like(d["x"])
    moe.moe_rmsnorm(d["x"], nw.cuda(), xn_gpu, EPS)
    c = run_chain(L, {**d, "x": xn_gpu})
    assert torch.equal(c["out"], r["out"])
    # the module wrapper with leading dims runs the same call
    mlp = moe.InklingMoE(inputs, E, k, S, w.route_scale, w.global_scale, norm_weight=nw,
                         norm_eps=EPS)
    m = mlp(d["x"].reshape(1, T, H)).reshape(T, H)
    assert torch.equal(m.cpu(), r["out"])


def test_forward_prenorm_full_size():
    w = mw.by_name("bf16-T8192-H6144-E128k8S1-I2048")
    inputs = mw.generate(w)
    nw = mw.norm_weight(w.H, seed=w.seed)
    r, _, _ = run_prenorm(w, inputs, nw, down_f16=True)
    xn = oracle.rmsnorm(inputs["x"], nw, EPS, out_dtype=w.torch_dtype)
    stats, _ = check_all(w, {**inputs, "x": xn}, r, strict=True)   # every token
    print(f"prenorm {w.name}: all {w.T} tokens, max|out - oracle| / RMS = {stats['rel_err']:.4f}; "
          f"{stats}")


def test_dense_prenorm():
    w = mw.dense_tiny(T=517, H=384, I=320, dtype="bf16", seed=12)
    inputs = mw.generate_dense(w)
    nw = mw.norm_weight(w.H, seed=5)
    mlp = moe.InklingDenseMLP(inputs["w_gate_up"], inputs["w_down"], norm_weight=nw, norm_eps=EPS)
    out = mlp(inputs["x"].cuda())
    torch.cuda.synchronize()
    xn = oracle.rmsnorm(inputs["x"], nw, EPS, out_dtype=torch.bfloat16)
    ref = oracle.dense_mlp(xn, inputs["w_gate_up"], inputs["w_down"], 1.0)
    check_output(out.cpu(), ref, torch.bfloat16, "dense prenorm out", strict=False)
