"""moe_permute_noalloc, the permutation for callers that cannot allocate
device memory (an engine plugin whose memory is planned ahead, a process on a
fixed memory budget): it keeps its counters in a static device array instead
of a caller workspace.  Its outputs must equal moe_permute's, call after call,
since each call starts from the previous call's leftover counters.

This file is collected last so that a failure here leaves every other test
already run; it also passes when run alone in a fresh process.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import moe_workloads as mw

pytestmark = pytest.mark.gpu


def _buffers(T, k, E, H, dtype):
    dev = "cuda"
    return (torch.full((E + 1,), -5, dtype=torch.int32, device=dev),
            torch.full((T * k,), -5, dtype=torch.int32, device=dev),
            torch.full((T * k,), -5, dtype=torch.int32, device=dev),
            torch.zeros(T * k, H, dtype=dtype, device=dev))


def _noalloc_call(lib, L, idx, pm, x, bufs, stream):
    off, ps, ip, xp = bufs
    return lib.moe_permute_noalloc(
        ctypes.byref(L.desc()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(pm.data_ptr()) if pm is not None else None,
        ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(off.data_ptr()),
        ctypes.c_void_p(ps.data_ptr()), ctypes.c_void_p(ip.data_ptr()),
        ctypes.c_void_p(xp.data_ptr()), ctypes.c_void_p(stream))


@pytest.mark.parametrize("T,H,E,k,pad", [(300, 256, 12, 3, False), (1000, 128, 64, 6, True),
                                         (70000, 64, 256, 8, True)])   # 1094 chunks of 512 slots
def test_noalloc_permute_matches_workspace_permute_twice(T, H, E, k, pad):
    import mixture_experts_feed_b200 as moe
    w = mw.tiny(T=T, H=H, E=E, k=k, S=1, I=64, dtype="bf16", seed=31)
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
        R = int(ref[0][-1])
        assert torch.equal(got[0], ref[0]), f"call {call}: expert_offsets differ"
        assert torch.equal(got[1][:R], ref[1][:R]), f"call {call}: perm_slot differs"
        assert torch.equal(got[2], ref[2]), f"call {call}: inv_perm differs"
        assert torch.equal(got[3][:R], ref[3][:R]), f"call {call}: x_perm differs"


def test_noalloc_permute_rejects_too_many_experts():
    import mixture_experts_feed_b200 as moe
    L = moe.Layer(8, 128, 1025, 2, 0, 64)      # E beyond the static array (and the library)
    fake = 1 << 20
    st = moe.LIB.moe_permute_noalloc(ctypes.byref(L.desc()), fake, None, fake, fake, fake, fake,
                                     fake, None)
    assert st == 2   # MOE_ERR_UNSUPPORTED
