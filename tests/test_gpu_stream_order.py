"""Stream order of the library's calls.

Every kernel of the layer is launched with programmatic stream
serialisation: its CTAs may start while the kernel before it on the stream
is still finishing, and they read or write global memory only once that
kernel has completed.  These tests queue calls and PyTorch kernels back to
back on one stream, with no host synchronisation between them, and check
that every result has the bits of the same call made alone after a full
synchronisation: a read that came too early would see the previous inputs,
a write that came too early would change a buffer a queued kernel was still
reading.
"""
from __future__ import annotations

import pytest
import torch

import moe_workloads as mw
from moe_gpu_helpers import down_f16_of, to_device

pytestmark = pytest.mark.gpu

try:
    import mixture_experts_feed_b200 as moe
except ImportError:   # collected on CPU-only machines too; the gpu marker deselects
    moe = None

SHAPES = [
    # T, H, E, k, S, I, dtype
    (300, 256, 12, 3, 2, 320, "bf16"),    # two shared experts: the side stream of moe_forward
    (1024, 4096, 8, 2, 1, 128, "bf16"),   # long K: the gate_up pair launch draws its tiles
    (77, 192, 10, 2, 3, 192, "f32"),      # fp32 layer (CUDA-core GEMMs)
]
IDS = ["bf16-S2", "bf16-H4096", "f32"]


def _case(T, H, E, k, S, I, dtype):
    """A layer (bf16 layers with fp16 down projections), its inputs on the GPU
    (x is input A) and a second input B."""
    w = mw.tiny(T=T, H=H, E=E, k=k, S=S, I=I, dtype=dtype, route_scale=2.5, seed=31)
    d = to_device(mw.generate(w, threads=4), down_f16=down_f16_of(w))
    gen = torch.Generator().manual_seed(32)
    xb = torch.randn(T, H, generator=gen).to(w.torch_dtype).cuda()
    return w, d, xb, moe.Layer.from_workload(w, down_f16=down_f16_of(w))


def _forward(L, d, x, out, ws, norm=None):
    S = L.S
    args = (d["w_router"], d["corr_bias"], d["w_gate_up"], d["w_down"],
            d["ws_gate_up"] if S else None, d["ws_down"] if S else None, out, ws)
    if norm is None:
        moe.moe_forward(L, x, *args)
    else:
        moe.moe_forward_prenorm(L, x, norm, 1e-6, *args)


@pytest.mark.parametrize("prenorm", [False, True], ids=["plain", "prenorm"])
@pytest.mark.parametrize("shape", SHAPES, ids=IDS)
def test_forward_calls_queued_back_to_back(shape, prenorm):
    """moe_forward on inputs A, B, A, B through one input buffer that a
    PyTorch copy refills before each call, a PyTorch clone of an output just
    before a call overwrites it, all on one stream without a host sync."""
    w, d, xb, L = _case(*shape)
    xa = d["x"]
    norm = None
    if prenorm:
        gen = torch.Generator().manual_seed(33)
        norm = (1.0 + 0.1 * torch.randn(w.H, generator=gen)).to(w.torch_dtype).cuda()
    ws = moe.new_workspace(L)
    ref = {}
    for name, x in (("a", xa), ("b", xb)):
        o = torch.empty(w.T, w.H, dtype=w.torch_dtype, device="cuda")
        _forward(L, d, x.clone(), o, ws, norm)
        torch.cuda.synchronize()
        ref[name] = o.clone()
    assert not torch.equal(ref["a"], ref["b"])

    xbuf = torch.full_like(xa, float("nan"))
    outs = [torch.full_like(ref["a"], float("nan")) for _ in range(3)]
    xbuf.copy_(xa)
    _forward(L, d, xbuf, outs[0], ws, norm)
    xbuf.copy_(xb)
    _forward(L, d, xbuf, outs[1], ws, norm)
    xbuf.copy_(xa)
    _forward(L, d, xbuf, outs[2], ws, norm)
    snapshot = outs[2].clone()       # read by PyTorch, then overwritten by the next call
    xbuf.copy_(xb)
    _forward(L, d, xbuf, outs[2], ws, norm)
    torch.cuda.synchronize()
    assert moe.read_device_status(ws) == 0
    assert torch.equal(outs[0], ref["a"])
    assert torch.equal(outs[1], ref["b"])
    assert torch.equal(snapshot, ref["a"])
    assert torch.equal(outs[2], ref["b"])


@pytest.mark.parametrize("shape", SHAPES[:2], ids=IDS[:2])
def test_op_chain_with_pytorch_kernels_between_calls(shape):
    """moe_route, moe_permute, moe_expert_ffn and moe_combine each read a
    buffer that a PyTorch kernel wrote just before the call on the same
    stream: the routing of B replaces that of A between route and permute,
    and B's permuted rows replace A's between permute and the GEMMs."""
    w, d, xb, L = _case(*shape)
    T, k, S, H, E = w.T, w.k, w.S, w.H, w.E
    ws = moe.new_workspace(L)
    dev = "cuda"

    def buffers():
        return {
            "tw": torch.empty(T, k, device=dev), "ti": torch.empty(T, k, dtype=torch.int32, device=dev),
            "sg": torch.empty(T, S, device=dev) if S else None,
            "off": torch.empty(E + 1, dtype=torch.int32, device=dev),
            "ps": torch.empty(T * k, dtype=torch.int32, device=dev),
            "ip": torch.empty(T * k, dtype=torch.int32, device=dev),
            "xp": torch.empty(T * k, H, dtype=L.dtype, device=dev),
            "yr": torch.empty(T * k, H, dtype=L.y_dtype, device=dev),
            "ys": torch.empty(S * T, H, dtype=L.y_dtype, device=dev) if S else None,
            "out": torch.empty(T, H, dtype=L.dtype, device=dev),
        }

    def route(x, b):
        moe.moe_route(L, x, d["w_router"], d["corr_bias"], b["tw"], b["ti"], b["sg"], ws)

    def permute(x, b):
        moe.moe_permute(L, b["ti"], None, x, b["off"], b["ps"], b["ip"], b["xp"], ws)

    def ffn(x, b):
        moe.moe_expert_ffn(L, x, b["xp"], b["off"], b["ps"], b["tw"], b["sg"], d["w_gate_up"],
                           d["w_down"], d["ws_gate_up"] if S else None,
                           d["ws_down"] if S else None, b["yr"], b["ys"], ws)

    def combine(b):
        moe.moe_combine(L, b["yr"], b["ys"], b["ip"], b["out"], ws)

    # references, each step synchronised
    ra, rb = buffers(), buffers()
    for x, b in ((d["x"], ra), (xb, rb)):
        for step in (route, permute, ffn):
            step(x, b)
            torch.cuda.synchronize()
        combine(b)
        torch.cuda.synchronize()

    # queued: routing of A, then PyTorch copies B's routing over it
    q = buffers()
    route(d["x"], q)
    q["tw"].copy_(rb["tw"])
    q["ti"].copy_(rb["ti"])
    if S:
        q["sg"].copy_(rb["sg"])
    permute(d["x"], q)                # B's order, A's rows ...
    q["xp"].copy_(rb["xp"])           # ... replaced by B's rows by PyTorch
    ffn(xb, q)
    combine(q)
    torch.cuda.synchronize()
    assert moe.read_device_status(ws) == 0
    for name in ("off", "ps", "ip", "xp", "yr", "out"):
        assert torch.equal(q[name], rb[name]), name
    if S:
        assert torch.equal(q["ys"], rb["ys"])


def test_dense_calls_queued_back_to_back():
    """moe_dense_mlp (gate_up and down with K split four ways at T = 32,
    whole-K tiles at T = 512) on inputs A, B, A through one buffer PyTorch
    refills before each call, without a host sync."""
    for T, H, I in ((32, 4096, 1024), (512, 512, 768)):
        w = mw.DenseWorkload(name=f"dense-bf16-T{T}-H{H}-I{I}", T=T, H=H, I=I, dtype="bf16",
                             global_scale=1.0, seed=34, init_std=0.02)
        d = to_device(mw.generate_dense(w, threads=4), down_f16=True)
        L = moe.DenseLayer.from_workload(w, down_f16=True)
        ws = moe.new_dense_workspace(L)
        gen = torch.Generator().manual_seed(35)
        xb = torch.randn(T, H, generator=gen).to(torch.bfloat16).cuda()
        ref = {}
        for name, x in (("a", d["x"]), ("b", xb)):
            o = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
            moe.moe_dense_mlp(L, x.clone(), d["w_gate_up"], d["w_down"], o, ws)
            torch.cuda.synchronize()
            ref[name] = o.clone()
        xbuf = torch.full_like(d["x"], float("nan"))
        outs = [torch.full_like(ref["a"], float("nan")) for _ in range(3)]
        for x, o in zip((d["x"], xb, d["x"]), outs):
            xbuf.copy_(x)
            moe.moe_dense_mlp(L, xbuf, d["w_gate_up"], d["w_down"], o, ws)
        torch.cuda.synchronize()
        assert moe.read_device_status(ws) == 0
        assert torch.equal(outs[0], ref["a"]) and torch.equal(outs[2], ref["a"])
        assert torch.equal(outs[1], ref["b"])


def _replay_matches_eager(call, x_static, out, make_x):
    """Capture call(x_static, out) in a CUDA graph, then replay it on new
    inputs and compare each replay bitwise with the eager call."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call(x_static, out)              # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(x_static, out)
    for i in range(3):
        x_new = make_x(i)
        x_static.copy_(x_new)
        g.replay()
        eager = torch.empty_like(out)
        call(x_new, eager)
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    del g


def test_chained_launches_in_cuda_graphs():
    """The pre-norm layer (norm, then the side stream of moe_forward) and the
    dense layer at T = 32 (K-split gate_up, SwiGLU pass, K-split down,
    recombination: four chained launches) captured in CUDA graphs replay
    with the eager calls' bits on new inputs."""
    w, d, xb, L = _case(300, 256, 12, 3, 2, 320, "bf16")
    gen = torch.Generator().manual_seed(36)
    norm = (1.0 + 0.1 * torch.randn(w.H, generator=gen)).to(torch.bfloat16).cuda()
    ws = moe.new_workspace(L)

    def moe_call(x, o):
        _forward(L, d, x, o, ws, norm)

    _replay_matches_eager(moe_call, d["x"].clone(), torch.empty_like(d["x"]),
                          lambda i: torch.randn(w.T, w.H, generator=gen).to(torch.bfloat16).cuda())
    assert moe.read_device_status(ws) == 0

    dw = mw.DenseWorkload(name="dense-bf16-T32-H4096-I1024", T=32, H=4096, I=1024, dtype="bf16",
                          global_scale=1.0, seed=37, init_std=0.02)
    dd = to_device(mw.generate_dense(dw, threads=4), down_f16=True)
    DL = moe.DenseLayer.from_workload(dw, down_f16=True)
    dws = moe.new_dense_workspace(DL)

    def dense_call(x, o):
        moe.moe_dense_mlp(DL, x, dd["w_gate_up"], dd["w_down"], o, dws)

    _replay_matches_eager(dense_call, dd["x"].clone(), torch.empty_like(dd["x"]),
                          lambda i: torch.randn(dw.T, dw.H, generator=gen).to(torch.bfloat16).cuda())
    assert moe.read_device_status(dws) == 0
