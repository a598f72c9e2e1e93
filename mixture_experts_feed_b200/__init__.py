"""Python binding of libinklingmoe.so, the B200 Inkling MoE feed-forward.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams.  The entry points keep
the C names (``moe_route``, ``moe_permute``, ``moe_expert_ffn``,
``moe_combine``, ``moe_forward``) and take torch tensors whose data pointers
are handed to the C ABI unchanged; shapes, dtypes and contiguity are checked
here so that a mistake raises instead of reaching the GPU.

There is no CPU fallback: importing this package raises when the shared
library has not been built (``python mixture_experts_feed_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libinklingmoe.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing; build it with `python mixture_experts_feed_b200/build.py`")

LIB = ctypes.CDLL(_LIB_PATH)
LIB_PATH = _LIB_PATH

MOE_F32, MOE_BF16, MOE_BF16_F16DOWN = 0, 1, 2
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_CHECK", 6: "MOE_ERR_TIMEOUT"}


class LayerDesc(ctypes.Structure):
    """``moe_layer_desc_t``."""
    _fields_ = [("num_tokens", ctypes.c_int64), ("hidden", ctypes.c_int32),
                ("n_routed", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("intermediate", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("route_scale", ctypes.c_float),
                ("global_scale", ctypes.c_float)]


class DenseDesc(ctypes.Structure):
    """``moe_dense_desc_t``."""
    _fields_ = [("num_tokens", ctypes.c_int64), ("hidden", ctypes.c_int32),
                ("intermediate", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("global_scale", ctypes.c_float)]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = LIB.moe_status_string(status).decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


_P = ctypes.c_void_p
_DESC = ctypes.POINTER(LayerDesc)
LIB.moe_status_string.restype = ctypes.c_char_p
LIB.moe_status_string.argtypes = [ctypes.c_int]
LIB.moe_version.restype = ctypes.c_int32
LIB.moe_forward_kernel_count.restype = ctypes.c_int32
LIB.moe_forward_kernel_count.argtypes = [_DESC]
LIB.moe_workspace_size.argtypes = [_DESC, ctypes.POINTER(ctypes.c_size_t)]
LIB.moe_workspace_init.argtypes = [_P, ctypes.c_size_t, _P]
LIB.moe_read_device_status.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_int32)]
LIB.moe_route.argtypes = [_DESC, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
LIB.moe_permute.argtypes = [_DESC, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
LIB.moe_permute_noalloc.argtypes = [_DESC, _P, _P, _P, _P, _P, _P, _P, _P]
LIB.moe_expert_ffn.argtypes = [_DESC] + [_P] * 13 + [ctypes.c_size_t, _P]
LIB.moe_combine.argtypes = [_DESC, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
LIB.moe_shared_ffn.argtypes = [_DESC, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
LIB.moe_shared_ffn_kernel_count.restype = ctypes.c_int32
LIB.moe_shared_ffn_kernel_count.argtypes = [_DESC]
LIB.moe_ep_dispatch_prep.argtypes = [_DESC, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
LIB.moe_ep_dispatch_p2p.argtypes = [_DESC, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P,
                                    ctypes.c_int64, _P, ctypes.c_size_t, _P]
LIB.moe_ep_return_p2p.argtypes = [_DESC, _P, ctypes.c_int64, _P, _P, ctypes.c_int32, _P,
                                  ctypes.c_int64, _P, ctypes.c_size_t, _P]
LIB.moe_convert_bf16_to_f16.argtypes = [ctypes.c_int64, _P, _P, _P, _P]
LIB.moe_forward.argtypes = [_DESC] + [_P] * 13 + [ctypes.c_size_t, _P]
LIB.moe_selftest_wait_timeout.argtypes = [_P, ctypes.c_size_t, ctypes.c_uint32, _P]
_DDESC = ctypes.POINTER(DenseDesc)
LIB.moe_dense_workspace_size.argtypes = [_DDESC, ctypes.POINTER(ctypes.c_size_t)]
LIB.moe_dense_mlp.argtypes = [_DDESC, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
LIB.moe_dense_kernel_count.restype = ctypes.c_int32
LIB.moe_dense_kernel_count.argtypes = [_DDESC]
LIB.moe_rmsnorm.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                            _P, _P, _P, _P]
LIB.moe_forward_prenorm.argtypes = [_DESC, _P, _P, ctypes.c_float] + [_P] * 12 + [ctypes.c_size_t, _P]
LIB.moe_dense_mlp_prenorm.argtypes = [_DDESC, _P, _P, ctypes.c_float, _P, _P, _P, _P,
                                      ctypes.c_size_t, _P]
LIB.moe_forward_prenorm_kernel_count.restype = ctypes.c_int32
LIB.moe_forward_prenorm_kernel_count.argtypes = [_DESC]
LIB.moe_dense_prenorm_kernel_count.restype = ctypes.c_int32
LIB.moe_dense_prenorm_kernel_count.argtypes = [_DDESC]
for _f in ("moe_workspace_size", "moe_workspace_init", "moe_read_device_status", "moe_route",
           "moe_permute", "moe_permute_noalloc", "moe_expert_ffn", "moe_combine", "moe_forward",
           "moe_selftest_wait_timeout", "moe_dense_workspace_size", "moe_dense_mlp",
           "moe_rmsnorm", "moe_forward_prenorm", "moe_dense_mlp_prenorm", "moe_shared_ffn",
           "moe_ep_dispatch_prep", "moe_ep_dispatch_p2p", "moe_ep_return_p2p",
           "moe_convert_bf16_to_f16"):
    getattr(LIB, _f).restype = ctypes.c_int


@dataclass(frozen=True)
class Layer:
    """Sizes and scales of one Inkling MoE layer (the ``InklingTextConfig`` MoE fields)."""
    T: int
    H: int
    E: int
    k: int
    S: int
    I: int
    dtype: torch.dtype = torch.bfloat16
    route_scale: float = 1.0
    global_scale: float = 1.0
    # bf16 layers only: the down projections' weights are fp16 copies and the
    # activated rows are rounded to fp16 (MOE_BF16_F16DOWN)
    down_f16: bool = False

    def desc(self) -> LayerDesc:
        return LayerDesc(self.T, self.H, self.E, self.k, self.S, self.I,
                         _layer_code(self.dtype, self.down_f16), self.route_scale, self.global_scale)

    @property
    def down_dtype(self) -> torch.dtype:
        """dtype of w_down / ws_down."""
        return torch.float16 if self.down_f16 else self.dtype

    @property
    def y_dtype(self) -> torch.dtype:
        """dtype of the expert output rows y_routed / y_shared."""
        return torch.float16 if self.down_f16 else torch.float32

    @staticmethod
    def from_workload(w, down_f16: bool = False) -> "Layer":
        return Layer(w.T, w.H, w.E, w.k, w.S, w.I, w.torch_dtype, w.route_scale, w.global_scale,
                     down_f16)


@dataclass(frozen=True)
class DenseLayer:
    """Sizes of the dense feed-forward layer (``InklingDenseMLP``)."""
    T: int
    H: int
    I: int
    dtype: torch.dtype = torch.bfloat16
    global_scale: float = 1.0
    down_f16: bool = False          # bf16 only: w_down fp16, activated rows fp16

    def desc(self) -> DenseDesc:
        return DenseDesc(self.T, self.H, self.I, _layer_code(self.dtype, self.down_f16),
                         self.global_scale)

    @property
    def down_dtype(self) -> torch.dtype:
        return torch.float16 if self.down_f16 else self.dtype

    @staticmethod
    def from_workload(w, down_f16: bool = False) -> "DenseLayer":
        return DenseLayer(w.T, w.H, w.I, w.torch_dtype, w.global_scale, down_f16)


def _layer_code(dtype: torch.dtype, down_f16: bool) -> int:
    if dtype == torch.float32 and not down_f16:
        return MOE_F32
    if dtype == torch.bfloat16:
        return MOE_BF16_F16DOWN if down_f16 else MOE_BF16
    raise ValueError(f"unsupported layer dtype {dtype} (down_f16={down_f16})")


def _check(status: int, where: str) -> None:
    if status != 0:
        raise MoEError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _expect(t: Optional[torch.Tensor], name: str, shape, dtype, allow_none=False) -> None:
    if t is None:
        if allow_none:
            return
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype} != {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    # the library launches on the current device: a buffer of another GPU
    # would be read through peer memory, or fault
    current = torch.cuda.current_device()
    if t.device.index != current:
        raise ValueError(f"{name} is on {t.device}, the current device is cuda:{current}")


def _wsptr(ws: torch.Tensor) -> int:
    """Device address of a workspace (a contiguous CUDA byte tensor of the
    current device)."""
    if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8 or not ws.is_contiguous():
        raise ValueError("the workspace must be a contiguous torch.uint8 tensor")
    if not ws.is_cuda or ws.device.index != torch.cuda.current_device():
        raise ValueError(f"the workspace is on {ws.device}, not on the current CUDA device")
    return ws.data_ptr()


def workspace_size(layer: Layer) -> int:
    n = ctypes.c_size_t(0)
    _check(LIB.moe_workspace_size(ctypes.byref(layer.desc()), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def new_workspace(layer: Layer, device=None, stream=None) -> torch.Tensor:
    """Allocate (with torch) and initialise a workspace for ``layer``."""
    ws = torch.empty(workspace_size(layer), dtype=torch.uint8, device=device or "cuda")
    _check(LIB.moe_workspace_init(_wsptr(ws), ws.numel(), _stream(stream)), "moe_workspace_init")
    return ws


def read_device_status(ws: torch.Tensor, stream=None) -> int:
    """Read and clear the device status word; raises MoEError when it is set."""
    code = ctypes.c_int32(0)
    st = LIB.moe_read_device_status(_wsptr(ws), _stream(stream), ctypes.byref(code))
    if st != 0:
        err = MoEError(st, f"device status 0x{code.value:x}")
        err.device_code = code.value
        raise err
    return code.value


def moe_route(layer: Layer, x, w_router, corr_bias, topk_w, topk_idx, shared_gamma, ws, stream=None):
    L = layer
    _expect(x, "x", (L.T, L.H), L.dtype)
    _expect(w_router, "w_router", (L.E + L.S, L.H), torch.float32)
    _expect(corr_bias, "corr_bias", (L.E,), torch.float32)
    _expect(topk_w, "topk_w", (L.T, L.k), torch.float32)
    _expect(topk_idx, "topk_idx", (L.T, L.k), torch.int32)
    _expect(shared_gamma, "shared_gamma", (L.T, L.S), torch.float32, allow_none=L.S == 0)
    _check(LIB.moe_route(ctypes.byref(L.desc()), _ptr(x), _ptr(w_router), _ptr(corr_bias),
                         _ptr(topk_w), _ptr(topk_idx), _ptr(shared_gamma), _wsptr(ws),
                         ws.numel(), _stream(stream)), "moe_route")


def moe_permute(layer: Layer, topk_idx, padding_mask, x, expert_offsets, perm_slot, inv_perm,
                x_perm, ws, stream=None):
    L = layer
    _expect(topk_idx, "topk_idx", (L.T, L.k), torch.int32)
    _expect(padding_mask, "padding_mask", (L.T,), torch.uint8, allow_none=True)
    _expect(x, "x", (L.T, L.H), L.dtype, allow_none=x_perm is None)
    _expect(expert_offsets, "expert_offsets", (L.E + 1,), torch.int32)
    _expect(perm_slot, "perm_slot", (L.T * L.k,), torch.int32)
    _expect(inv_perm, "inv_perm", (L.T * L.k,), torch.int32)
    _expect(x_perm, "x_perm", (L.T * L.k, L.H), L.dtype, allow_none=True)   # None: no row copy
    _check(LIB.moe_permute(ctypes.byref(L.desc()), _ptr(topk_idx), _ptr(padding_mask), _ptr(x),
                           _ptr(expert_offsets), _ptr(perm_slot), _ptr(inv_perm), _ptr(x_perm),
                           _wsptr(ws), ws.numel(), _stream(stream)), "moe_permute")


def moe_permute_noalloc(layer: Layer, topk_idx, padding_mask, x, expert_offsets, perm_slot,
                        inv_perm, x_perm, stream=None):
    """``moe_permute`` without a workspace, for callers that cannot allocate
    device memory (its scratch is a static device array; E <= 1024; calls
    that overlap on the GPU race on that array)."""
    L = layer
    _expect(topk_idx, "topk_idx", (L.T, L.k), torch.int32)
    _expect(padding_mask, "padding_mask", (L.T,), torch.uint8, allow_none=True)
    _expect(x, "x", (L.T, L.H), L.dtype, allow_none=x_perm is None)
    _expect(expert_offsets, "expert_offsets", (L.E + 1,), torch.int32)
    _expect(perm_slot, "perm_slot", (L.T * L.k,), torch.int32)
    _expect(inv_perm, "inv_perm", (L.T * L.k,), torch.int32)
    _expect(x_perm, "x_perm", (L.T * L.k, L.H), L.dtype, allow_none=True)   # None: no row copy
    _check(LIB.moe_permute_noalloc(ctypes.byref(L.desc()), _ptr(topk_idx), _ptr(padding_mask),
                                   _ptr(x), _ptr(expert_offsets), _ptr(perm_slot), _ptr(inv_perm),
                                   _ptr(x_perm), _stream(stream)), "moe_permute_noalloc")


def moe_expert_ffn(layer: Layer, x, x_perm, expert_offsets, perm_slot, topk_w, shared_gamma,
                   w_gate_up, w_down, ws_gate_up, ws_down, y_routed, y_shared, ws, stream=None):
    L = layer
    _expect(x, "x", (L.T, L.H), L.dtype)
    # None: the gate_up GEMM gathers the routed rows of x through perm_slot
    _expect(x_perm, "x_perm", (L.T * L.k, L.H), L.dtype, allow_none=True)
    _expect(expert_offsets, "expert_offsets", (L.E + 1,), torch.int32)
    # perm_slot None (with x_perm given): the rows are already in slot order
    _expect(perm_slot, "perm_slot", (L.T * L.k,), torch.int32, allow_none=x_perm is not None)
    if topk_w.numel() != L.T * L.k or topk_w.dtype != torch.float32 or not topk_w.is_contiguous():
        raise ValueError("topk_w must be a contiguous fp32 tensor of T*k entries")
    if L.S > 0 and (shared_gamma is None or shared_gamma.numel() != L.T * L.S):
        raise ValueError("shared_gamma must hold T*S entries")
    _expect(w_gate_up, "w_gate_up", (L.E, 2 * L.I, L.H), L.dtype)
    _expect(w_down, "w_down", (L.E, L.H, L.I), L.down_dtype)
    _expect(ws_gate_up, "ws_gate_up", (L.S, 2 * L.I, L.H), L.dtype, allow_none=L.S == 0)
    _expect(ws_down, "ws_down", (L.S, L.H, L.I), L.down_dtype, allow_none=L.S == 0)
    _expect(y_routed, "y_routed", (L.T * L.k, L.H), L.y_dtype)
    _expect(y_shared, "y_shared", (L.S * L.T, L.H), L.y_dtype, allow_none=L.S == 0)
    _check(LIB.moe_expert_ffn(ctypes.byref(L.desc()), _ptr(x), _ptr(x_perm), _ptr(expert_offsets),
                              _ptr(perm_slot), _ptr(topk_w), _ptr(shared_gamma), _ptr(w_gate_up),
                              _ptr(w_down), _ptr(ws_gate_up), _ptr(ws_down), _ptr(y_routed),
                              _ptr(y_shared), _wsptr(ws), ws.numel(), _stream(stream)),
           "moe_expert_ffn")


def moe_shared_ffn(layer: Layer, x, shared_gamma, ws_gate_up, ws_down, y_shared, ws, stream=None):
    """The shared experts alone (``InklingSharedExperts.forward``): y_shared
    rows s*T + t in fp32."""
    L = layer
    _expect(x, "x", (L.T, L.H), L.dtype)
    _expect(shared_gamma, "shared_gamma", (L.T, L.S), torch.float32)
    _expect(ws_gate_up, "ws_gate_up", (L.S, 2 * L.I, L.H), L.dtype)
    _expect(ws_down, "ws_down", (L.S, L.H, L.I), L.down_dtype)
    _expect(y_shared, "y_shared", (L.S * L.T, L.H), L.y_dtype)
    _check(LIB.moe_shared_ffn(ctypes.byref(L.desc()), _ptr(x), _ptr(shared_gamma),
                              _ptr(ws_gate_up), _ptr(ws_down), _ptr(y_shared), _wsptr(ws),
                              ws.numel(), _stream(stream)), "moe_shared_ffn")


def shared_ffn_kernel_count(layer: Layer) -> int:
    return int(LIB.moe_shared_ffn_kernel_count(ctypes.byref(layer.desc())))


def moe_ep_dispatch_prep(layer: Layer, expert_offsets, perm_slot, topk_w, row_w, expert_counts,
                         ws, stream=None):
    """Routing weight of every permuted row and the per-expert row counts
    (the sending side of expert parallelism)."""
    L = layer
    _expect(expert_offsets, "expert_offsets", (L.E + 1,), torch.int32)
    _expect(perm_slot, "perm_slot", (L.T * L.k,), torch.int32)
    if topk_w.numel() != L.T * L.k or topk_w.dtype != torch.float32 or not topk_w.is_contiguous():
        raise ValueError("topk_w must be a contiguous fp32 tensor of T*k entries")
    _expect(row_w, "row_w", (L.T * L.k,), torch.float32)
    _expect(expert_counts, "expert_counts", (L.E,), torch.int32)
    _check(LIB.moe_ep_dispatch_prep(ctypes.byref(L.desc()), _ptr(expert_offsets), _ptr(perm_slot),
                                    _ptr(topk_w), _ptr(row_w), _ptr(expert_counts), _wsptr(ws),
                                    ws.numel(), _stream(stream)), "moe_ep_dispatch_prep")


def _ptr_table(ptrs, n: int, what: str) -> None:
    if (not isinstance(ptrs, torch.Tensor) or ptrs.dtype != torch.int64 or ptrs.numel() != n
            or not ptrs.is_cuda or not ptrs.is_contiguous()):
        raise ValueError(f"{what} must be a contiguous int64 CUDA tensor of {n} device pointers")


def moe_ep_dispatch_p2p(layer: Layer, x, topk_w, perm_slot, expert_offsets, dst_base, n_ranks: int,
                        dst_x, dst_w, dst_rows: int, ws, stream=None):
    """Every permuted row of this rank, with its weight, stored straight into
    the receive buffers of the rank that owns its expert (``dst_x`` /
    ``dst_w``: int64 CUDA tensors of ``n_ranks`` device pointers, buffers of
    ``dst_rows`` rows; ``dst_base [E]``: where this rank's rows of each expert
    start there)."""
    L = layer
    _expect(x, "x", (L.T, L.H), L.dtype)
    if topk_w.numel() != L.T * L.k or topk_w.dtype != torch.float32 or not topk_w.is_contiguous():
        raise ValueError("topk_w must be a contiguous fp32 tensor of T*k entries")
    _expect(perm_slot, "perm_slot", (L.T * L.k,), torch.int32)
    _expect(expert_offsets, "expert_offsets", (L.E + 1,), torch.int32)
    _expect(dst_base, "dst_base", (L.E,), torch.int32)
    _ptr_table(dst_x, n_ranks, "dst_x")
    _ptr_table(dst_w, n_ranks, "dst_w")
    _check(LIB.moe_ep_dispatch_p2p(ctypes.byref(L.desc()), _ptr(x), _ptr(topk_w), _ptr(perm_slot),
                                   _ptr(expert_offsets), _ptr(dst_base), n_ranks, _ptr(dst_x),
                                   _ptr(dst_w), dst_rows, _wsptr(ws), ws.numel(),
                                   _stream(stream)), "moe_ep_dispatch_p2p")


def moe_ep_return_p2p(layer: Layer, y_in, rows_in: int, run_start, src_base, n_ranks: int, dst_y,
                      dst_rows: int, ws, stream=None):
    """Every received output row stored straight into its source's y rows
    (``dst_y``: int64 CUDA tensor of ``n_ranks`` device pointers to buffers of
    ``dst_rows`` rows); runs ordered by local expert, then source."""
    L = layer
    if y_in.dtype != L.y_dtype or y_in.dim() != 2 or y_in.shape[1] != L.H or y_in.shape[0] < rows_in \
            or not y_in.is_contiguous():
        raise ValueError(f"y_in must be a contiguous [>= {rows_in}, {L.H}] {L.y_dtype} tensor")
    _expect(run_start, "run_start", (L.E + 1,), torch.int32)
    _expect(src_base, "src_base", (L.E,), torch.int32)
    _ptr_table(dst_y, n_ranks, "dst_y")
    _check(LIB.moe_ep_return_p2p(ctypes.byref(L.desc()), _ptr(y_in), rows_in, _ptr(run_start),
                                 _ptr(src_base), n_ranks, _ptr(dst_y), dst_rows, _wsptr(ws),
                                 ws.numel(), _stream(stream)), "moe_ep_return_p2p")


def moe_combine(layer: Layer, y_routed, y_shared, inv_perm, out, ws, stream=None):
    L = layer
    _expect(y_routed, "y_routed", (L.T * L.k, L.H), L.y_dtype)
    _expect(y_shared, "y_shared", (L.S * L.T, L.H), L.y_dtype, allow_none=L.S == 0)
    _expect(inv_perm, "inv_perm", (L.T * L.k,), torch.int32)
    _expect(out, "out", (L.T, L.H), L.dtype)
    _check(LIB.moe_combine(ctypes.byref(L.desc()), _ptr(y_routed), _ptr(y_shared), _ptr(inv_perm),
                           _ptr(out), _wsptr(ws), ws.numel(), _stream(stream)), "moe_combine")


def moe_forward(layer: Layer, x, w_router, corr_bias, w_gate_up, w_down, ws_gate_up, ws_down,
                out, ws, padding_mask=None, topk_w=None, topk_idx=None, shared_gamma=None,
                stream=None):
    L = layer
    _expect(x, "x", (L.T, L.H), L.dtype)
    _expect(w_router, "w_router", (L.E + L.S, L.H), torch.float32)
    _expect(corr_bias, "corr_bias", (L.E,), torch.float32)
    _expect(w_gate_up, "w_gate_up", (L.E, 2 * L.I, L.H), L.dtype)
    _expect(w_down, "w_down", (L.E, L.H, L.I), L.down_dtype)
    _expect(ws_gate_up, "ws_gate_up", (L.S, 2 * L.I, L.H), L.dtype, allow_none=L.S == 0)
    _expect(ws_down, "ws_down", (L.S, L.H, L.I), L.down_dtype, allow_none=L.S == 0)
    _expect(out, "out", (L.T, L.H), L.dtype)
    _expect(padding_mask, "padding_mask", (L.T,), torch.uint8, allow_none=True)
    _expect(topk_w, "topk_w", (L.T, L.k), torch.float32, allow_none=True)
    _expect(topk_idx, "topk_idx", (L.T, L.k), torch.int32, allow_none=True)
    _expect(shared_gamma, "shared_gamma", (L.T, L.S), torch.float32, allow_none=True)
    _check(LIB.moe_forward(ctypes.byref(L.desc()), _ptr(x), _ptr(w_router), _ptr(corr_bias),
                           _ptr(w_gate_up), _ptr(w_down), _ptr(ws_gate_up), _ptr(ws_down),
                           _ptr(padding_mask), _ptr(out), _ptr(topk_w), _ptr(topk_idx),
                           _ptr(shared_gamma), _wsptr(ws), ws.numel(), _stream(stream)),
           "moe_forward")


def _dtype_code(dtype: torch.dtype) -> int:
    code = {torch.float32: MOE_F32, torch.bfloat16: MOE_BF16}.get(dtype)
    if code is None:
        raise ValueError(f"unsupported dtype {dtype}")
    return code


def moe_rmsnorm(x, weight, out, eps: float = 1e-6, stream=None):
    """``InklingRMSNorm``: ``x`` [T, H] -> ``out`` [T, H] (may be ``x``)."""
    if x.dim() != 2:
        raise ValueError("x must be [T, H]")
    T, H = x.shape
    _expect(x, "x", (T, H), x.dtype)
    _expect(weight, "weight", (H,), x.dtype)
    _expect(out, "out", (T, H), x.dtype)
    _check(LIB.moe_rmsnorm(T, H, _dtype_code(x.dtype), eps, _ptr(x), _ptr(weight), _ptr(out),
                           _stream(stream)), "moe_rmsnorm")


def moe_forward_prenorm(layer: Layer, x, norm_weight, norm_eps, w_router, corr_bias, w_gate_up,
                        w_down, ws_gate_up, ws_down, out, ws, padding_mask=None, topk_w=None,
                        topk_idx=None, shared_gamma=None, stream=None):
    L = layer
    _expect(norm_weight, "norm_weight", (L.H,), L.dtype)
    _expect(x, "x", (L.T, L.H), L.dtype)
    _expect(w_router, "w_router", (L.E + L.S, L.H), torch.float32)
    _expect(corr_bias, "corr_bias", (L.E,), torch.float32)
    _expect(w_gate_up, "w_gate_up", (L.E, 2 * L.I, L.H), L.dtype)
    _expect(w_down, "w_down", (L.E, L.H, L.I), L.down_dtype)
    _expect(ws_gate_up, "ws_gate_up", (L.S, 2 * L.I, L.H), L.dtype, allow_none=L.S == 0)
    _expect(ws_down, "ws_down", (L.S, L.H, L.I), L.down_dtype, allow_none=L.S == 0)
    _expect(out, "out", (L.T, L.H), L.dtype)
    _expect(padding_mask, "padding_mask", (L.T,), torch.uint8, allow_none=True)
    _expect(topk_w, "topk_w", (L.T, L.k), torch.float32, allow_none=True)
    _expect(topk_idx, "topk_idx", (L.T, L.k), torch.int32, allow_none=True)
    _expect(shared_gamma, "shared_gamma", (L.T, L.S), torch.float32, allow_none=True)
    _check(LIB.moe_forward_prenorm(ctypes.byref(L.desc()), _ptr(x), _ptr(norm_weight), norm_eps,
                                   _ptr(w_router), _ptr(corr_bias), _ptr(w_gate_up), _ptr(w_down),
                                   _ptr(ws_gate_up), _ptr(ws_down), _ptr(padding_mask), _ptr(out),
                                   _ptr(topk_w), _ptr(topk_idx), _ptr(shared_gamma), _wsptr(ws),
                                   ws.numel(), _stream(stream)), "moe_forward_prenorm")


def moe_dense_mlp_prenorm(layer: "DenseLayer", x, norm_weight, norm_eps, w_gate_up, w_down, out,
                          ws, stream=None):
    L = layer
    _expect(norm_weight, "norm_weight", (L.H,), L.dtype)
    _expect(x, "x", (L.T, L.H), L.dtype)
    _expect(w_gate_up, "w_gate_up", (2 * L.I, L.H), L.dtype)
    _expect(w_down, "w_down", (L.H, L.I), L.down_dtype)
    _expect(out, "out", (L.T, L.H), L.dtype)
    _check(LIB.moe_dense_mlp_prenorm(ctypes.byref(L.desc()), _ptr(x), _ptr(norm_weight), norm_eps,
                                     _ptr(w_gate_up), _ptr(w_down), _ptr(out), _wsptr(ws),
                                     ws.numel(), _stream(stream)), "moe_dense_mlp_prenorm")


def forward_prenorm_kernel_count(layer: Layer) -> int:
    return int(LIB.moe_forward_prenorm_kernel_count(ctypes.byref(layer.desc())))


def dense_prenorm_kernel_count(layer: "DenseLayer") -> int:
    return int(LIB.moe_dense_prenorm_kernel_count(ctypes.byref(layer.desc())))


def selftest_wait_timeout(ws: torch.Tensor, limit_ms: int = 1000, stream=None) -> None:
    """Launch the stall-detection self-test (see the header); the next
    read_device_status() raises MoEError with MOE_ERR_TIMEOUT."""
    _check(LIB.moe_selftest_wait_timeout(_wsptr(ws), ws.numel(), limit_ms, _stream(stream)),
           "moe_selftest_wait_timeout")


def forward_kernel_count(layer: Layer) -> int:
    return int(LIB.moe_forward_kernel_count(ctypes.byref(layer.desc())))


def dense_workspace_size(layer: DenseLayer) -> int:
    n = ctypes.c_size_t(0)
    _check(LIB.moe_dense_workspace_size(ctypes.byref(layer.desc()), ctypes.byref(n)),
           "moe_dense_workspace_size")
    return n.value


def new_dense_workspace(layer: DenseLayer, device=None, stream=None) -> torch.Tensor:
    """Allocate (with torch) and initialise a workspace for the dense ``layer``."""
    ws = torch.empty(dense_workspace_size(layer), dtype=torch.uint8, device=device or "cuda")
    _check(LIB.moe_workspace_init(_wsptr(ws), ws.numel(), _stream(stream)), "moe_workspace_init")
    return ws


def moe_dense_mlp(layer: DenseLayer, x, w_gate_up, w_down, out, ws, stream=None):
    L = layer
    _expect(x, "x", (L.T, L.H), L.dtype)
    _expect(w_gate_up, "w_gate_up", (2 * L.I, L.H), L.dtype)
    _expect(w_down, "w_down", (L.H, L.I), L.down_dtype)
    _expect(out, "out", (L.T, L.H), L.dtype)
    _check(LIB.moe_dense_mlp(ctypes.byref(L.desc()), _ptr(x), _ptr(w_gate_up), _ptr(w_down),
                             _ptr(out), _wsptr(ws), ws.numel(), _stream(stream)),
           "moe_dense_mlp")


def dense_kernel_count(layer: DenseLayer) -> int:
    return int(LIB.moe_dense_kernel_count(ctypes.byref(layer.desc())))


def convert_bf16_to_f16(src: torch.Tensor, out: Optional[torch.Tensor] = None,
                        nonfinite: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``moe_convert_bf16_to_f16``: the fp16 copy of bf16 down-projection
    weights (for layers with ``down_f16``), asynchronous; ``nonfinite`` (an
    int32 CUDA tensor of one element) counts the elements with no finite fp16
    value."""
    if src.dtype != torch.bfloat16 or not src.is_contiguous() or not src.is_cuda:
        raise ValueError("src must be a contiguous bf16 CUDA tensor")
    out = torch.empty(src.shape, dtype=torch.float16, device=src.device) if out is None else out
    _expect(out, "out", tuple(src.shape), torch.float16)
    if nonfinite is not None:
        _expect(nonfinite, "nonfinite", (1,), torch.int32)
    _check(LIB.moe_convert_bf16_to_f16(src.numel(), _ptr(src), _ptr(out), _ptr(nonfinite),
                                       _stream(stream)), "moe_convert_bf16_to_f16")
    return out


def prepare_down_weights(w_down: torch.Tensor, stream=None) -> torch.Tensor:
    """The fp16 copy of one bf16 down-projection weight tensor (exact for
    magnitudes from 2^-17 to 65504; smaller ones change by at most 2^-25);
    raises ValueError when an element has no finite fp16 value (synchronises
    ``stream``)."""
    count = torch.zeros(1, dtype=torch.int32, device=w_down.device)
    out = convert_bf16_to_f16(w_down.contiguous(), nonfinite=count, stream=stream)
    n = int(count.item())
    if n:
        raise ValueError(f"{n} down-projection weights have no finite fp16 value")
    return out


class InklingMoE:
    """Device-resident weights of one layer plus its workspace; ``__call__``
    runs ``moe_forward`` on ``x`` of shape ``[..., H]`` (leading dims are
    flattened to tokens, as ``InklingMoE.forward`` does)."""

    def __init__(self, weights: dict, E: int, k: int, S: int, route_scale: float,
                 global_scale: float = 1.0, device="cuda", norm_weight=None, norm_eps: float = 1e-6):
        self.w = {n: t.to(device).contiguous() for n, t in weights.items() if n != "x"}
        # optional post_attention_layernorm run first (moe_forward_prenorm)
        self.norm_weight = None if norm_weight is None else norm_weight.to(device).contiguous()
        self.norm_eps = norm_eps
        self.E, self.k, self.S = E, k, S
        self.H = self.w["w_router"].shape[1]
        self.I = self.w["w_down"].shape[2]
        self.dtype = self.w["w_gate_up"].dtype
        # fp16 down weights (from prepare_down_weights): fp16 down projections
        self.down_f16 = self.w["w_down"].dtype == torch.float16
        self.route_scale, self.global_scale = route_scale, global_scale
        self.device = device
        self._ws = None
        self._ws_T = -1

    def layer(self, T: int) -> Layer:
        return Layer(T, self.H, self.E, self.k, self.S, self.I, self.dtype, self.route_scale,
                     self.global_scale, self.down_f16)

    def __call__(self, x: torch.Tensor, padding_mask: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        lead = x.shape[:-1]
        xt = x.reshape(-1, self.H).contiguous()
        L = self.layer(xt.shape[0])
        if self._ws is None or self._ws_T < L.T:
            self._ws = new_workspace(L, device=self.device, stream=stream)
            self._ws_T = L.T
        out = torch.empty_like(xt)
        pm = None
        if padding_mask is not None:
            pm = padding_mask.reshape(-1).to(device=xt.device, dtype=torch.uint8).contiguous()
        w = self.w
        wsgu = w.get("ws_gate_up") if self.S else None
        wsd = w.get("ws_down") if self.S else None
        if self.norm_weight is None:
            moe_forward(L, xt, w["w_router"], w["corr_bias"], w["w_gate_up"], w["w_down"], wsgu,
                        wsd, out, self._ws, padding_mask=pm, stream=stream)
        else:
            moe_forward_prenorm(L, xt, self.norm_weight, self.norm_eps, w["w_router"],
                                w["corr_bias"], w["w_gate_up"], w["w_down"], wsgu, wsd, out,
                                self._ws, padding_mask=pm, stream=stream)
        return out.reshape(*lead, self.H)


class InklingDenseMLP:
    """Device-resident weights of the dense feed-forward layer plus its
    workspace; ``__call__`` runs ``moe_dense_mlp`` on ``x`` of shape
    ``[..., H]`` (leading dims flattened to tokens)."""

    def __init__(self, w_gate_up: torch.Tensor, w_down: torch.Tensor, global_scale: float = 1.0,
                 device="cuda", norm_weight=None, norm_eps: float = 1e-6):
        # optional post_attention_layernorm run first (moe_dense_mlp_prenorm)
        self.norm_weight = None if norm_weight is None else norm_weight.to(device).contiguous()
        self.norm_eps = norm_eps
        self.w_gate_up = w_gate_up.to(device).contiguous()
        self.w_down = w_down.to(device).contiguous()
        self.H = self.w_gate_up.shape[1]
        self.I = self.w_down.shape[1]
        self.dtype = self.w_gate_up.dtype
        self.down_f16 = self.w_down.dtype == torch.float16
        self.global_scale = global_scale
        self.device = device
        self._ws = None
        self._ws_T = -1

    def layer(self, T: int) -> DenseLayer:
        return DenseLayer(T, self.H, self.I, self.dtype, self.global_scale, self.down_f16)

    def __call__(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        lead = x.shape[:-1]
        xt = x.reshape(-1, self.H).contiguous()
        L = self.layer(xt.shape[0])
        if self._ws is None or self._ws_T < L.T:
            self._ws = new_dense_workspace(L, device=self.device, stream=stream)
            self._ws_T = L.T
        out = torch.empty_like(xt)
        if self.norm_weight is None:
            moe_dense_mlp(L, xt, self.w_gate_up, self.w_down, out, self._ws, stream=stream)
        else:
            moe_dense_mlp_prenorm(L, xt, self.norm_weight, self.norm_eps, self.w_gate_up,
                                  self.w_down, out, self._ws, stream=stream)
        return out.reshape(*lead, self.H)
