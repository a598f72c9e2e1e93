"""The C-ABI library loads on a machine without a GPU, exports every entry
point the header declares, and rejects bad arguments on the host before any
CUDA call.  No compute call is made here."""
from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

import mixture_experts_feed_b200 as moe
import moe_workloads as mw

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "inkling_moe.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_five_ops():
    names = declared_functions()
    for f in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward",
              "moe_workspace_size"):
        assert f in names


def test_library_exports_every_declared_symbol():
    for name in declared_functions():
        assert hasattr(moe.LIB, name), f"{name} not exported by {moe.LIB_PATH}"


def test_version_and_strings():
    assert moe.LIB.moe_version() >= 1
    for code in range(7):
        assert moe.LIB.moe_status_string(code)


def test_desc_struct_layout_matches_header():
    # int64 + 6 x int32 + 2 x float, naturally aligned
    assert ctypes.sizeof(moe.LayerDesc) == 40
    assert moe.LayerDesc.route_scale.offset == 32


@pytest.mark.parametrize("w", mw.ORDERED, ids=[w.name for w in mw.ORDERED])
def test_workspace_size_covers_intermediates(w):
    L = moe.Layer.from_workload(w)
    n = moe.workspace_size(L)
    el = 4 if w.dtype == "f32" else 2
    Rk = w.T * w.k
    need = el * (Rk * w.H + (Rk + w.S * w.T) * w.I) + 4 * (Rk + w.S * w.T) * w.H
    assert n >= need
    # bf16: gate_up and down as CTA-pair + single-CTA launches (T > 128), and
    # with shared experts their own gate_up on moe_forward's side stream (their
    # down joins the routed experts' down launches)
    experts = ((4 if w.T > 128 else 2) + (1 if w.S else 0)) if w.dtype == "bf16" else 2
    # tensor-core router: K split across ~148 CTAs when T is small; from 4
    # splits on, below 2048 tokens, a separate kernel sums the partial logits
    # before the top-k
    ksplit = 1
    if w.dtype == "bf16":
        tiles = -(-w.T // 128) * -(-(w.E + w.S) // 160)
        ksplit = max(1, min(32, 148 // tiles))
    router = (2 if w.dtype == "bf16" else 1) + (2 if ksplit >= 4 and w.T < 2048 else 1)
    # permute: chunk counts, chunk scan, scatter, row gather (at most 256
    # slots: one kernel for the first three)
    permute = 2 if w.T * w.k <= 256 else 4
    assert moe.forward_kernel_count(L) == router + permute + experts + 1


def _status(fn, *args):
    return getattr(moe.LIB, fn)(*args)


def test_invalid_descriptors_are_rejected():
    n = ctypes.c_size_t(0)
    bad = [
        moe.Layer(4, 128, 8, 0, 1, 64),        # k = 0
        moe.Layer(4, 128, 8, 9, 1, 64),        # k > E
        moe.Layer(-1, 128, 8, 2, 1, 64),       # T < 0
        moe.Layer(4, 0, 8, 2, 1, 64),          # H = 0
    ]
    for L in bad:
        assert _status("moe_workspace_size", ctypes.byref(L.desc()), ctypes.byref(n)) == 1
    unsupported = [
        moe.Layer(4, 100, 8, 2, 1, 64),        # H not a multiple of 64
        moe.Layer(4, 128, 8, 2, 1, 48),        # I not a multiple of 64
        moe.Layer(4, 128, 2048, 2, 1, 64),     # E > 1024
        moe.Layer(4, 128, 64, 17, 1, 64),      # k > 16
        moe.Layer(4, 128, 8, 2, 9, 64),        # S > 8
        moe.Layer(2**26 + 1, 128, 8, 2, 1, 64),  # T > 2^26 (with k + S <= 24, T * (k + S) < 2^31)
    ]
    for L in unsupported:
        assert _status("moe_workspace_size", ctypes.byref(L.desc()), ctypes.byref(n)) == 2
    assert _status("moe_workspace_size", None, ctypes.byref(n)) == 1
    assert _status("moe_workspace_size", ctypes.byref(moe.Layer(4, 128, 8, 2, 1, 64).desc()), None) == 1


def test_null_and_misaligned_pointers_are_rejected_before_launch():
    L = moe.Layer(16, 128, 8, 2, 1, 64)
    d = ctypes.byref(L.desc())
    fake = 1 << 20          # aligned, never dereferenced: the checks fail first
    ws_ok = moe.workspace_size(L)
    # null x
    assert _status("moe_route", d, None, fake, fake, fake, fake, fake, fake, ws_ok, None) == 1
    # misaligned x
    assert _status("moe_route", d, fake + 2, fake, fake, fake, fake, fake, fake, ws_ok, None) == 1
    # missing gamma with S > 0
    assert _status("moe_route", d, fake, fake, fake, fake, fake, None, fake, ws_ok, None) == 1
    # workspace too small
    assert _status("moe_route", d, fake, fake, fake, fake, fake, fake, fake, ws_ok - 1, None) == 3
    # workspace misaligned
    assert _status("moe_route", d, fake, fake, fake, fake, fake, fake, fake + 16, ws_ok, None) == 1
    assert _status("moe_permute", d, None, None, fake, fake, fake, fake, fake, fake, ws_ok, None) == 1
    assert _status("moe_expert_ffn", d, fake, fake, fake, fake, fake, None, fake, fake, fake, fake,
                   fake, fake, fake, ws_ok, None) == 1
    assert _status("moe_combine", d, fake, fake, fake, None, fake, ws_ok, None) == 1
    assert _status("moe_forward", d, fake, fake, fake, fake, fake, None, fake, None, fake,
                   None, None, None, fake, ws_ok, None) == 1
    assert _status("moe_workspace_init", None, 1024, None) == 1
    assert _status("moe_selftest_wait_timeout", None, 1024, 100, None) == 1
    assert _status("moe_selftest_wait_timeout", fake, 1024, 0, None) == 1
    assert _status("moe_read_device_status", None, None, None) == 1


def test_noalloc_permute_host_checks():
    L = moe.Layer(16, 128, 8, 2, 1, 64)
    d = ctypes.byref(L.desc())
    fake = 1 << 20          # aligned, never dereferenced: the checks fail first
    f = moe.LIB.moe_permute_noalloc
    assert f(d, None, None, fake, fake, fake, fake, fake, None) == 1          # no topk_idx
    assert f(d, fake, None, None, fake, fake, fake, fake, None) == 1          # a copy needs x
    assert f(d, fake, None, fake + 8, fake, fake, fake, fake, None) == 1      # misaligned x
    assert f(d, fake, None, fake, fake, fake, fake, fake + 4, None) == 1      # misaligned x_perm
    assert f(d, fake, None, fake, fake, None, fake, fake, None) == 1          # no perm_slot


def test_binding_checks_shapes_on_host():
    L = moe.Layer(4, 128, 8, 2, 1, 64, torch.float32)
    x = torch.zeros(4, 64)   # wrong H, on CPU: rejected before the C call
    with pytest.raises(ValueError):
        moe.moe_combine(L, x, x, torch.zeros(8, dtype=torch.int32), x, torch.zeros(16, dtype=torch.uint8))


def test_binding_rejects_a_buffer_of_another_device(monkeypatch):
    """Every op launches on the current device; a tensor on another GPU is
    rejected on the host (checked with a stand-in object: no GPU here)."""
    from types import SimpleNamespace
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    other = SimpleNamespace(shape=(4, 128), dtype=torch.float32, is_contiguous=lambda: True,
                            is_cuda=True, device=torch.device("cuda", 1))
    with pytest.raises(ValueError, match="current device"):
        moe._expect(other, "x", (4, 128), torch.float32)
    same = SimpleNamespace(shape=(4, 128), dtype=torch.float32, is_contiguous=lambda: True,
                           is_cuda=True, device=torch.device("cuda", 0))
    moe._expect(same, "x", (4, 128), torch.float32)


# ------------------------------------------------------------- dense layer
def test_dense_desc_layout_and_sizes():
    assert ctypes.sizeof(moe.DenseDesc) == 24     # int64 + 3 x int32 + float
    assert moe.DenseDesc.global_scale.offset == 20
    for w in mw.DENSE_WORKLOADS.values():
        L = moe.DenseLayer.from_workload(w)
        el = 4 if w.dtype == "f32" else 2
        assert moe.dense_workspace_size(L) >= el * w.T * w.I + 4 * w.T * w.H
        # gate_up, down, rounding pass; a weight-streaming bf16 layer with few
        # tokens (decode) splits gate_up's K and adds the SwiGLU pass over the splits
        split = w.dtype == "bf16" and w.T <= 32 and w.H >= 2048
        assert moe.dense_kernel_count(L) == (4 if split else 3)
        if split:   # room for the K-split accumulators [ks, T, 2I] fp32
            assert moe.dense_workspace_size(L) >= el * w.T * w.I + 4 * w.T * w.H + 2 * 4 * w.T * 2 * w.I
    for T in (0, 1, 32, 129):              # host-side tiling choices at the edges
        for dt in (torch.bfloat16, torch.float32):
            assert moe.dense_workspace_size(moe.DenseLayer(T, 128, 64, dt)) > 0
    assert moe.dense_kernel_count(moe.DenseLayer(0, 128, 64)) == 0


def _dense_status(T=8, H=64, I=64, dtype=moe.MOE_BF16, gs=1.0, ws_bytes=None, ptr=256):
    d = moe.DenseDesc(T, H, I, dtype, gs)
    if ws_bytes is None:
        ws_bytes = 1 << 40     # large enough for any valid desc; argument checks come first
    # aligned fake pointers: every call below returns on the host before any
    # CUDA call, so nothing is dereferenced
    return moe.LIB.moe_dense_mlp(ctypes.byref(d), ptr, ptr, ptr, ptr, 4096, ws_bytes, None)


def test_dense_host_checks():
    assert _dense_status(H=100) == 2                      # H % 64
    assert _dense_status(I=96) == 2                       # I % 64
    assert _dense_status(T=-1) == 1
    assert _dense_status(gs=float("nan")) == 1
    assert _dense_status(dtype=7) == 1
    assert _dense_status(ws_bytes=100) == 3               # workspace too small
    assert _dense_status(ptr=8) == 1                      # misaligned operand
    assert _dense_status(T=0, ptr=0) == 0                 # T = 0: nothing read
    assert moe.LIB.moe_dense_workspace_size(None, None) == 1


def test_dense_binding_checks_shapes():
    L = moe.DenseLayer(4, 64, 64)
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moe.moe_dense_mlp(L, x, torch.zeros(64, 64, dtype=torch.bfloat16),     # not [2I, H]
                          torch.zeros(64, 64, dtype=torch.bfloat16), x, None)


def declared_arity():
    """Parameter count of every function the header declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(moe_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", src):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argtypes_match_the_header():
    """Every ctypes prototype the binding sets has the header's parameter
    count (a missing argument shifts the rest, which ctypes does not catch)."""
    arity = declared_arity()
    assert len(arity) == len(declared_functions())
    for name, n in arity.items():
        fn = getattr(moe.LIB, name)
        if fn.argtypes is None:
            assert n == 0, f"{name}: no ctypes prototype for {n} parameters"
        else:
            assert len(fn.argtypes) == n, f"{name}: {len(fn.argtypes)} argtypes, header has {n}"


def test_new_entry_points_host_checks():
    """moe_shared_ffn and moe_ep_dispatch_prep reject bad arguments on the
    host, before any CUDA call (fake aligned pointers are never touched)."""
    fake, big = 1 << 20, 1 << 40
    L = moe.Layer(64, 128, 8, 2, 0, 64)                      # no shared expert
    d = ctypes.byref(L.desc())
    assert moe.LIB.moe_shared_ffn(d, fake, fake, fake, fake, fake, fake, big, None) == 1
    L1 = moe.Layer(64, 128, 8, 2, 1, 64)
    d1 = ctypes.byref(L1.desc())
    assert moe.LIB.moe_shared_ffn(d1, fake + 8, fake, fake, fake, fake, fake, big, None) == 1   # misaligned x
    assert moe.LIB.moe_shared_ffn(d1, fake, None, fake, fake, fake, fake, big, None) == 1       # no gammas
    assert moe.LIB.moe_shared_ffn(d1, fake, fake, fake, fake, fake, fake, 100, None) == 3       # workspace
    assert moe.LIB.moe_shared_ffn_kernel_count(d1) == 2
    assert moe.LIB.moe_shared_ffn_kernel_count(d) == 0
    L0 = moe.Layer(0, 128, 8, 2, 1, 64)
    assert moe.LIB.moe_shared_ffn(ctypes.byref(L0.desc()), fake, fake, fake, fake, fake, fake, big,
                                  None) == 0                 # T = 0: nothing launched
    for i in range(5):                                        # each required pointer null in turn
        args = [fake] * 5
        args[i] = None
        assert moe.LIB.moe_ep_dispatch_prep(d1, *args, fake, 4096, None) == 1
    assert moe.LIB.moe_ep_dispatch_prep(d1, fake, fake, fake, fake, fake, fake + 16, 4096, None) == 1
    assert moe.LIB.moe_ep_dispatch_prep(d1, fake, fake, fake, fake, fake, fake, 100, None) == 1


def test_peer_memory_entry_points_host_checks():
    """moe_ep_dispatch_p2p and moe_ep_return_p2p reject bad arguments on the
    host (fake aligned pointers are never touched)."""
    fake, big = 1 << 20, 1 << 40
    L = moe.Layer(64, 128, 8, 2, 1, 64)
    d = ctypes.byref(L.desc())
    ok = [fake, fake, fake, fake, fake]                       # x, topk_w, perm_slot, offsets, dst_base
    for i in range(5):
        args = list(ok)
        args[i] = None
        assert moe.LIB.moe_ep_dispatch_p2p(d, *args, 2, fake, fake, 100, fake, 4096, None) == 1
    assert moe.LIB.moe_ep_dispatch_p2p(d, fake + 8, *ok[1:], 2, fake, fake, 100, fake, 4096, None) == 1
    assert moe.LIB.moe_ep_dispatch_p2p(d, *ok, 3, fake, fake, 100, fake, 4096, None) == 1   # 8 % 3
    assert moe.LIB.moe_ep_dispatch_p2p(d, *ok, 2, None, fake, 100, fake, 4096, None) == 1
    assert moe.LIB.moe_ep_dispatch_p2p(d, *ok, 2, fake, fake, 100, fake, 100, None) == 1   # workspace
    assert moe.LIB.moe_ep_return_p2p(d, fake, 10, None, fake, 2, fake, 100, fake, 4096, None) == 1
    assert moe.LIB.moe_ep_return_p2p(d, fake, 10, fake, fake, 0, fake, 100, fake, 4096, None) == 1
    assert moe.LIB.moe_ep_return_p2p(d, fake + 8, 10, fake, fake, 2, fake, 100, fake, 4096, None) == 1
    assert moe.LIB.moe_ep_return_p2p(d, fake, -1, fake, fake, 2, fake, 100, fake, 4096, None) == 1
    assert moe.LIB.moe_ep_return_p2p(d, None, 0, fake, fake, 2, fake, 100, fake, 4096, None) == 0
    L0 = moe.Layer(0, 128, 8, 2, 1, 64)
    assert moe.LIB.moe_ep_dispatch_p2p(ctypes.byref(L0.desc()), *ok, 2, fake, fake, 100, fake, 4096,
                                       None) == 0          # T = 0: nothing launched


def test_expert_ffn_needs_a_row_map_or_a_copy():
    """moe_expert_ffn takes perm_slot = NULL only when x_perm is given (rows
    already in slot order); with neither the rows cannot be found."""
    fake, big = 1 << 20, 1 << 40
    L = moe.Layer(64, 128, 8, 2, 0, 64)
    d = ctypes.byref(L.desc())
    args = [fake, None, fake, None, fake, None, fake, fake, None, None, fake, None]
    assert moe.LIB.moe_expert_ffn(d, *args, fake, big, None) == 1


def test_ep_partition():
    from mixture_experts_feed_b200.ep import partition
    assert partition(128, 8, 3) == (48, 16)
    with pytest.raises(ValueError):
        partition(10, 4, 0)


def test_convert_host_checks():
    """moe_convert_bf16_to_f16: n a multiple of 8, both buffers present and
    16-byte aligned; n = 0 does nothing."""
    fake = 1 << 20
    assert moe.LIB.moe_convert_bf16_to_f16(12, fake, fake, None, None) == 1       # n % 8
    assert moe.LIB.moe_convert_bf16_to_f16(-8, fake, fake, None, None) == 1
    assert moe.LIB.moe_convert_bf16_to_f16(16, None, fake, None, None) == 1
    assert moe.LIB.moe_convert_bf16_to_f16(16, fake, fake + 2, None, None) == 1   # misaligned
    assert moe.LIB.moe_convert_bf16_to_f16(0, None, None, None, None) == 0


def test_layer_codes():
    """The binding's layer dtypes map onto moe_dtype_t; fp16 down projections
    exist for bf16 layers only."""
    assert moe.Layer(4, 64, 4, 1, 0, 64, torch.bfloat16).desc().dtype == moe.MOE_BF16
    assert moe.Layer(4, 64, 4, 1, 0, 64, torch.bfloat16, down_f16=True).desc().dtype == moe.MOE_BF16_F16DOWN
    assert moe.Layer(4, 64, 4, 1, 0, 64, torch.float32).desc().dtype == moe.MOE_F32
    with pytest.raises(ValueError):
        moe.Layer(4, 64, 4, 1, 0, 64, torch.float32, down_f16=True).desc()
    L = moe.Layer(4, 64, 4, 1, 0, 64, torch.bfloat16, down_f16=True)
    assert L.down_dtype == torch.float16 and L.y_dtype == torch.float16
    # the workspace of a fp16-down layer holds fp16 expert rows: smaller
    Lb = moe.Layer(512, 256, 8, 2, 1, 128, torch.bfloat16)
    Lf = moe.Layer(512, 256, 8, 2, 1, 128, torch.bfloat16, down_f16=True)
    assert moe.workspace_size(Lf) < moe.workspace_size(Lb)
