"""moe_permute_noalloc, the permutation for callers that cannot allocate
device memory (an engine plugin whose memory is planned ahead, a process on a
fixed memory budget): it keeps its counters in a static device array instead
of a caller workspace.  Its outputs must equal moe_permute's and the
oracle's stable (expert, token) sort, call after call, since each call starts
from the previous call's leftover counters.

This file is collected last so that a failure here leaves every other test
already run; it also passes when run alone in a fresh process.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import moe_workloads as mw
import oracle

pytestmark = pytest.mark.gpu


def _buffers(T, k, E, H, dtype, with_copy=True):
    dev = "cuda"
    return (torch.full((E + 1,), -5, dtype=torch.int32, device=dev),
            torch.full((T * k,), -5, dtype=torch.int32, device=dev),
            torch.full((T * k,), -5, dtype=torch.int32, device=dev),
            torch.zeros(T * k, H, dtype=dtype, device=dev) if with_copy else None)


def _noalloc_call(lib, L, idx, pm, x, bufs, stream):
    """moe_permute_noalloc straight through the C ABI (ctypes)."""
    off, ps, ip, xp = bufs
    return lib.moe_permute_noalloc(
        ctypes.byref(L.desc()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(pm.data_ptr()) if pm is not None else None,
        ctypes.c_void_p(x.data_ptr()) if xp is not None else None,
        ctypes.c_void_p(off.data_ptr()), ctypes.c_void_p(ps.data_ptr()),
        ctypes.c_void_p(ip.data_ptr()),
        ctypes.c_void_p(xp.data_ptr()) if xp is not None else None, ctypes.c_void_p(stream))


def _check_against_oracle(got, idx, pm, x, k, E, call):
    """offsets, perm_slot, inv_perm bit-exact against the oracle's stable sort
    of the same ids and mask; x_perm rows equal to the tokens' rows of x."""
    off, ps, ip, xp = (t.cpu() if t is not None else None for t in got)
    ref = oracle.permute(idx.cpu().to(torch.int64), E, None if pm is None else pm.cpu())
    R = int(ref["offsets"][-1])
    assert torch.equal(off.to(torch.int64), ref["offsets"]), f"call {call}: offsets vs oracle"
    assert torch.equal(ps[:R].to(torch.int64), ref["perm_slot"]), f"call {call}: perm_slot vs oracle"
    assert torch.equal(ip.to(torch.int64), ref["inv_perm"]), f"call {call}: inv_perm vs oracle"
    if xp is not None:
        assert torch.equal(xp[:R], x.cpu()[ref["perm_slot"] // k]), f"call {call}: x_perm rows"
    return R


@pytest.mark.parametrize("T,H,E,k,pad,dtype", [
    (300, 256, 12, 3, False, "bf16"),
    (1000, 128, 64, 6, True, "bf16"),
    (70000, 64, 256, 8, True, "bf16"),     # 1094 chunks of 512 slots in moe_permute
    (517, 192, 40, 4, True, "f32"),        # fp32 rows in the gather
])
def test_noalloc_permute_matches_workspace_permute_twice(T, H, E, k, pad, dtype):
    import mixture_experts_feed_b200 as moe
    w = mw.tiny(T=T, H=H, E=E, k=k, S=1, I=64, dtype=dtype, seed=31)
    inputs = mw.generate(w, threads=2, with_experts=False)
    L = moe.Layer.from_workload(w)
    x = inputs["x"].cuda()
    g = torch.Generator().manual_seed(7)
    pm = (torch.rand(T, generator=g) < 0.2).to(torch.uint8).cuda() if pad else None
    stream = torch.cuda.current_stream().cuda_stream
    ws = moe.new_workspace(L)
    for call in range(2):
        # a different selection on each call: the second starts from the first's counters
        idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32).cuda()
        ref = _buffers(T, k, E, H, L.dtype)
        moe.moe_permute(L, idx, pm, x, *ref, ws)
        got = _buffers(T, k, E, H, L.dtype)
        assert _noalloc_call(moe.LIB, L, idx, pm, x, got, stream) == 0
        torch.cuda.synchronize()
        assert moe.read_device_status(ws) == 0
        R = _check_against_oracle(got, idx, pm, x, k, E, call)
        assert torch.equal(got[0], ref[0]), f"call {call}: expert_offsets differ"
        assert torch.equal(got[1][:R], ref[1][:R]), f"call {call}: perm_slot differs"
        assert torch.equal(got[2], ref[2]), f"call {call}: inv_perm differs"
        assert torch.equal(got[3][:R], ref[3][:R]), f"call {call}: x_perm differs"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_permute_binding_without_row_copy_twice(dtype):
    """The Python binding with x_perm = None (no row copy; x is then not
    passed at all): the index outputs still equal the oracle's sort and the
    workspace path's, on two calls in a row with different selections."""
    import mixture_experts_feed_b200 as moe
    T, H, E, k = 700, 128, 24, 4
    L = moe.Layer(T, H, E, k, 0, 64, torch.bfloat16 if dtype == "bf16" else torch.float32)
    g = torch.Generator().manual_seed(11)
    pm = (torch.rand(T, generator=g) < 0.15).to(torch.uint8).cuda()
    ws = moe.new_workspace(L)
    for call in range(2):
        idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32).cuda()
        got = _buffers(T, k, E, H, L.dtype, with_copy=False)
        moe.moe_permute_noalloc(L, idx, pm, None, got[0], got[1], got[2], None)
        ref = _buffers(T, k, E, H, L.dtype, with_copy=False)
        moe.moe_permute(L, idx, pm, None, ref[0], ref[1], ref[2], None, ws)
        torch.cuda.synchronize()
        assert moe.read_device_status(ws) == 0
        R = _check_against_oracle(got, idx, pm, None, k, E, call)
        assert torch.equal(got[0], ref[0]) and torch.equal(got[2], ref[2])
        assert torch.equal(got[1][:R], ref[1][:R])


def test_noalloc_permute_rejects_too_many_experts():
    import mixture_experts_feed_b200 as moe
    L = moe.Layer(8, 128, 1025, 2, 0, 64)      # E beyond the static array (and the library)
    fake = 1 << 20
    st = moe.LIB.moe_permute_noalloc(ctypes.byref(L.desc()), fake, None, fake, fake, fake, fake,
                                     fake, None)
    assert st == 2   # MOE_ERR_UNSUPPORTED
