"""ctypes binding of ``libep_b200.so`` (declared in ``include/ep_b200.h``).

Argument marshalling only: each function checks tensor dtypes, shapes and
devices, passes raw pointers and the current CUDA stream to the C entry point of
the same name, and raises :class:`EpError` on a non-zero status.  Every step of
the computation runs in the library's CUDA kernels; there is no fallback.  If
the library has not been built, importing this module raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libep_b200.so")

EP_OK, EP_ERR_INVALID_ARG, EP_ERR_SHAPE, EP_ERR_WORKSPACE, EP_ERR_CUDA = 0, 1, 2, 3, 4
EP_DEV_INDEX_RANGE, EP_DEV_TIMEOUT, EP_DEV_CAPACITY = 0x1, 0x2, 0x4
EP_QUANT_NONE, EP_QUANT_FP8_E4M3_1X128, EP_QUANT_FP8_E4M3_1X128_POW2 = 0, 1, 2
EP_QUANT_SCALES_MN_MAJOR = 0x100  # OR-ed into an FP8 quant: recv_scales [H/128, ld]


def scales_ld(rows: int) -> int:
    """Leading dimension of block-major (MN-major) scales for `rows` worst-case rows."""
    return (rows + 3) // 4 * 4


def _scale_numel(quant: int, rows: int, H: int) -> int:
    return (H // 128) * (scales_ld(rows) if quant & EP_QUANT_SCALES_MN_MAJOR else rows)

EXPORTED = (
    "ep_abi_version", "ep_status_string", "ep_workspace_bytes", "ep_workspace_init",
    "ep_read_status", "ep_get_dispatch_layout", "ep_dispatch", "ep_combine",
    "ep_low_latency_dispatch", "ep_low_latency_combine", "ep_debug_wait_probe",
    "ep_get_dispatch_layout_static", "ep_dispatch_backward", "ep_combine_backward",
    "ep_dispatch_dedup", "ep_combine_dedup", "ep_lb_prefetch_weights", "ep_lb_reduce_grads",
    "ep_ipc_alloc", "ep_ipc_free", "ep_ipc_open", "ep_ipc_close", "ep_peer_plan",
    "ep_peer_dispatch", "ep_peer_combine", "ep_get_dispatch_layout_dedup",
    "ep_peer_dispatch_dedup", "ep_peer_combine_dedup", "ep_peer_low_latency_dispatch",
    "ep_peer_low_latency_combine",
)
EP_IPC_HANDLE_BYTES = 64


class EpError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")
        self.status = status


class ep_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "num_tokens_per_expert", "num_tokens_per_partition", "is_token_in_partition",
        "expert_offset", "row_of", "src_of", "num_recv")]


class ep_ll_handle(ctypes.Structure):
    _fields_ = [("row_of", ctypes.c_void_p), ("src_of", ctypes.c_void_p)]


class ep_peer_buffers(ctypes.Structure):
    _fields_ = [("recv_x", ctypes.c_void_p), ("recv_scales", ctypes.c_void_p),
                ("recv_topk_idx", ctypes.c_void_p), ("recv_topk_weights", ctypes.c_void_p),
                ("capacity", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python combine_get_dispatch_05_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    i64, i32, sz, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t, ctypes.c_void_p
    st = ctypes.c_int32
    L.ep_abi_version.argtypes, L.ep_abi_version.restype = [], i32
    L.ep_status_string.argtypes, L.ep_status_string.restype = [i32], ctypes.c_char_p
    L.ep_workspace_bytes.argtypes, L.ep_workspace_bytes.restype = [i64, i32, i32], sz
    L.ep_workspace_init.argtypes, L.ep_workspace_init.restype = [vp, sz, vp], st
    L.ep_read_status.argtypes = [vp, sz, vp, ctypes.POINTER(ctypes.c_uint32)]
    L.ep_read_status.restype = st
    L.ep_get_dispatch_layout.argtypes = [i64, i32, i32, i32, vp, ctypes.POINTER(ep_layout), vp, sz,
                                         vp]
    L.ep_get_dispatch_layout.restype = st
    L.ep_dispatch.argtypes = [i64, i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp,
                              ctypes.POINTER(ep_layout), vp, sz, vp]
    L.ep_dispatch.restype = st
    L.ep_combine.argtypes = [i64, i64, i32, vp, i64, ctypes.POINTER(ep_layout), vp, vp, vp, sz, vp]
    L.ep_combine.restype = st
    L.ep_low_latency_dispatch.argtypes = [i64, i64, i32, i32, i32, vp, vp, vp, vp, vp,
                                          ctypes.POINTER(ep_ll_handle), vp, sz, vp]
    L.ep_low_latency_dispatch.restype = st
    L.ep_low_latency_combine.argtypes = [i64, i64, i32, i32, i32, vp,
                                         ctypes.POINTER(ep_ll_handle), vp, vp, vp, sz, vp]
    L.ep_low_latency_combine.restype = st
    L.ep_debug_wait_probe.argtypes, L.ep_debug_wait_probe.restype = [ctypes.c_uint64, vp, sz, vp], st
    L.ep_lb_prefetch_weights.argtypes = [i32, i64, vp, vp, vp, sz, vp]
    L.ep_lb_prefetch_weights.restype = st
    L.ep_lb_reduce_grads.argtypes = [i32, i64, vp, vp, vp, sz, vp]
    L.ep_lb_reduce_grads.restype = st
    L.ep_get_dispatch_layout_static.argtypes = [i64, i32, i32, i32, vp,
                                                ctypes.POINTER(ep_layout), vp]
    L.ep_get_dispatch_layout_static.restype = st
    L.ep_dispatch_backward.argtypes = [i64, i64, i32, vp, i64, ctypes.POINTER(ep_layout), vp, vp, vp,
                                       vp, sz, vp]
    L.ep_dispatch_backward.restype = st
    L.ep_combine_backward.argtypes = [i64, i64, i32, vp, vp, i64, ctypes.POINTER(ep_layout), vp, vp,
                                      vp, vp, sz, vp]
    L.ep_combine_backward.restype = st
    L.ep_dispatch_dedup.argtypes = [i64, i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp,
                                    ctypes.POINTER(ep_layout), vp, sz, vp]
    L.ep_dispatch_dedup.restype = st
    L.ep_combine_dedup.argtypes = [i64, i64, i32, vp, i64, ctypes.POINTER(ep_layout), vp, vp, sz,
                                   vp]
    L.ep_combine_dedup.restype = st
    L.ep_ipc_alloc.argtypes = [sz, ctypes.POINTER(vp), vp]
    L.ep_ipc_alloc.restype = st
    L.ep_ipc_free.argtypes, L.ep_ipc_free.restype = [vp], st
    L.ep_ipc_open.argtypes, L.ep_ipc_open.restype = [vp, ctypes.POINTER(vp)], st
    L.ep_ipc_close.argtypes, L.ep_ipc_close.restype = [vp], st
    L.ep_peer_plan.argtypes = [i32, i32, i32, vp, vp, i64, vp, vp, vp, vp, sz, vp]
    L.ep_peer_plan.restype = st
    L.ep_peer_dispatch.argtypes = [i64, i64, i32, i32, i32, i32, vp, vp, vp,
                                   ctypes.POINTER(ep_layout), vp, ctypes.POINTER(ep_peer_buffers),
                                   vp, sz, vp]
    L.ep_peer_dispatch.restype = st
    L.ep_peer_combine.argtypes = [i64, i64, i32, i32, i32, vp, i64, ctypes.POINTER(ep_layout), vp,
                                  vp, vp, vp, vp, sz, vp]
    L.ep_peer_combine.restype = st
    L.ep_get_dispatch_layout_dedup.argtypes = [i64, i32, i32, i32, vp, ctypes.POINTER(ep_layout),
                                               vp, sz, vp]
    L.ep_get_dispatch_layout_dedup.restype = st
    L.ep_peer_dispatch_dedup.argtypes = L.ep_peer_dispatch.argtypes
    L.ep_peer_dispatch_dedup.restype = st
    L.ep_peer_combine_dedup.argtypes = [i64, i64, i32, vp, i64, ctypes.POINTER(ep_layout), vp, vp,
                                        vp, sz, vp]
    L.ep_peer_combine_dedup.restype = st
    L.ep_peer_low_latency_dispatch.argtypes = [i64, i64, i32, i32, i32, i32, i32, vp, vp, vp, vp,
                                               vp, ctypes.POINTER(ep_ll_handle), vp, sz, vp]
    L.ep_peer_low_latency_dispatch.restype = st
    L.ep_peer_low_latency_combine.argtypes = [i64, i64, i32, i32, i32, i32, i32, vp, vp,
                                              ctypes.POINTER(ep_ll_handle), vp, vp, vp, sz, vp]
    L.ep_peer_low_latency_combine.restype = st
    return L


lib = _load()


def status_string(status: int) -> str:
    return lib.ep_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != EP_OK:
        raise EpError(fn, status)


# the current stream's handle without building a Stream object (a few us less per
# call); torch.cuda.current_stream() where this torch does not offer it
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream) -> int:
    if stream is None:
        if _raw_stream is not None:
            return _raw_stream(torch.cuda.current_device())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype, shape=None, numel_at_least=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if numel_at_least is not None and t.numel() < numel_at_least:
        raise ValueError(f"{name} needs at least {numel_at_least} elements, has {t.numel()}")


# ----------------------------------------------------------------- handles --

@dataclass
class Layout:
    """Device arrays of one batch's routing layout -- the `handle` that dispatch
    returns and combine consumes (see ``ep_layout`` in ep_b200.h)."""

    num_tokens_per_expert: torch.Tensor  # int32 [E]
    num_tokens_per_partition: torch.Tensor  # int32 [P]
    is_token_in_partition: torch.Tensor  # uint8 [T, P]
    expert_offset: torch.Tensor  # int32 [E + 1]
    row_of: torch.Tensor  # int32 [T, K]
    src_of: torch.Tensor  # int32 [T * K]
    num_recv: torch.Tensor  # int32 [1]

    @staticmethod
    def empty(num_tokens: int, num_topk: int, num_experts: int, num_partitions: int,
              device) -> "Layout":
        i32 = dict(dtype=torch.int32, device=device)
        return Layout(
            torch.empty(num_experts, **i32), torch.empty(num_partitions, **i32),
            torch.empty((num_tokens, num_partitions), dtype=torch.uint8, device=device),
            torch.empty(num_experts + 1, **i32), torch.empty((num_tokens, num_topk), **i32),
            torch.empty(max(num_tokens * num_topk, 1), **i32), torch.empty(1, **i32))

    def c(self) -> ep_layout:
        return ep_layout(*(t.data_ptr() for t in (
            self.num_tokens_per_expert, self.num_tokens_per_partition,
            self.is_token_in_partition, self.expert_offset, self.row_of, self.src_of,
            self.num_recv)))


@dataclass
class LowLatencyHandle:
    """Device arrays of a low-latency dispatch (see ``ep_ll_handle``)."""

    row_of: torch.Tensor  # int32 [T, K]: e * num_max_tokens + slot, or -1
    src_of: torch.Tensor  # int32 [E, num_max_tokens]
    num_max_tokens: int
    num_experts: int

    @staticmethod
    def empty(num_tokens: int, num_topk: int, num_experts: int, num_max_tokens: int,
              device) -> "LowLatencyHandle":
        return LowLatencyHandle(
            torch.empty((num_tokens, num_topk), dtype=torch.int32, device=device),
            torch.empty((num_experts, num_max_tokens), dtype=torch.int32, device=device),
            num_max_tokens, num_experts)

    def c(self) -> ep_ll_handle:
        return ep_ll_handle(self.row_of.data_ptr(), self.src_of.data_ptr())


# --------------------------------------------------------------- workspace --

def ep_workspace_bytes(num_tokens: int, num_experts: int, num_partitions: int) -> int:
    return int(lib.ep_workspace_bytes(num_tokens, num_experts, num_partitions))


def ep_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _need(workspace, "workspace", torch.uint8)
    _check("ep_workspace_init",
           lib.ep_workspace_init(workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_read_status(workspace: torch.Tensor, stream=None) -> int:
    _need(workspace, "workspace", torch.uint8)
    bits = ctypes.c_uint32(0)
    _check("ep_read_status", lib.ep_read_status(workspace.data_ptr(), workspace.numel(),
                                                _stream(stream), ctypes.byref(bits)))
    return int(bits.value)


# ---------------------------------------------------------------- calls -----

def ep_get_dispatch_layout(topk_idx: torch.Tensor, num_experts: int, num_partitions: int,
                           layout: Layout, workspace: torch.Tensor, stream=None) -> None:
    _need(topk_idx, "topk_idx", torch.int64)
    T, K = topk_idx.shape
    _need(layout.row_of, "layout.row_of", torch.int32, shape=(T, K))
    _need(layout.num_tokens_per_expert, "layout.num_tokens_per_expert", torch.int32,
          shape=(num_experts,))
    _need(layout.num_tokens_per_partition, "layout.num_tokens_per_partition", torch.int32,
          shape=(num_partitions,))
    _need(layout.is_token_in_partition, "layout.is_token_in_partition", torch.uint8,
          shape=(T, num_partitions))
    _need(layout.expert_offset, "layout.expert_offset", torch.int32, shape=(num_experts + 1,))
    _need(layout.src_of, "layout.src_of", torch.int32, numel_at_least=T * K)
    _need(workspace, "workspace", torch.uint8)
    c = layout.c()
    _check("ep_get_dispatch_layout", lib.ep_get_dispatch_layout(
        T, K, num_experts, num_partitions, topk_idx.data_ptr(), ctypes.byref(c),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                num_experts: int, num_partitions: int, quant: int, recv_x: torch.Tensor,
                recv_scales: Optional[torch.Tensor], recv_topk_idx: torch.Tensor,
                recv_topk_weights: torch.Tensor, handle: Layout, workspace: torch.Tensor,
                stream=None) -> None:
    _need(x, "x", torch.bfloat16)
    T, H = x.shape
    K = topk_idx.shape[1]
    _need(topk_idx, "topk_idx", torch.int64, shape=(T, K))
    _need(topk_weights, "topk_weights", torch.float32, shape=(T, K))
    if quant & ~EP_QUANT_SCALES_MN_MAJOR in (EP_QUANT_FP8_E4M3_1X128, EP_QUANT_FP8_E4M3_1X128_POW2):
        _need(recv_x, "recv_x", (torch.uint8, torch.float8_e4m3fn), numel_at_least=T * K * H)
        _need(recv_scales, "recv_scales", torch.float32,
              numel_at_least=_scale_numel(quant, T * K, H))
    else:
        _need(recv_x, "recv_x", torch.bfloat16, numel_at_least=T * K * H)
    _need(recv_topk_idx, "recv_topk_idx", torch.int32, numel_at_least=T * K)
    _need(recv_topk_weights, "recv_topk_weights", torch.float32, numel_at_least=T * K)
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, K))
    _need(handle.src_of, "handle.src_of", torch.int32, numel_at_least=T * K)
    _need(handle.is_token_in_partition, "handle.is_token_in_partition", torch.uint8,
          shape=(T, num_partitions))
    _need(handle.num_tokens_per_expert, "handle.num_tokens_per_expert", torch.int32,
          shape=(num_experts,))
    _need(handle.expert_offset, "handle.expert_offset", torch.int32, shape=(num_experts + 1,))
    _need(workspace, "workspace", torch.uint8)
    c = handle.c()
    _check("ep_dispatch", lib.ep_dispatch(
        T, H, K, num_experts, num_partitions, quant, x.data_ptr(), topk_idx.data_ptr(),
        topk_weights.data_ptr(), recv_x.data_ptr(), _ptr(recv_scales), recv_topk_idx.data_ptr(),
        recv_topk_weights.data_ptr(), ctypes.byref(c), workspace.data_ptr(), workspace.numel(),
        _stream(stream)))


def ep_combine(expert_out: torch.Tensor, handle: Layout, topk_weights: torch.Tensor,
               y: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    _need(expert_out, "expert_out", torch.bfloat16)
    H = expert_out.shape[-1]
    rows = expert_out.numel() // H if H else 0
    T, K = topk_weights.shape
    _need(topk_weights, "topk_weights", torch.float32)
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, K))
    _need(y, "y", torch.bfloat16, shape=(T, H))
    _need(workspace, "workspace", torch.uint8)
    c = ep_layout(row_of=handle.row_of.data_ptr())
    _check("ep_combine", lib.ep_combine(
        T, H, K, expert_out.data_ptr(), rows, ctypes.byref(c), topk_weights.data_ptr(),
        y.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_low_latency_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, num_max_tokens: int,
                            num_experts: int, recv_x: torch.Tensor, recv_scales: torch.Tensor,
                            recv_expert_count: torch.Tensor, handle: LowLatencyHandle,
                            workspace: torch.Tensor, stream=None) -> None:
    _need(x, "x", torch.bfloat16)
    T, H = x.shape
    K = topk_idx.shape[1]
    _need(topk_idx, "topk_idx", torch.int64, shape=(T, K))
    _need(recv_x, "recv_x", (torch.uint8, torch.float8_e4m3fn),
          shape=(num_experts, num_max_tokens, H))
    _need(recv_scales, "recv_scales", torch.float32,
          shape=(num_experts, num_max_tokens, H // 128))
    _need(recv_expert_count, "recv_expert_count", torch.int32, shape=(num_experts,))
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, K))
    _need(handle.src_of, "handle.src_of", torch.int32, shape=(num_experts, num_max_tokens))
    _need(workspace, "workspace", torch.uint8)
    c = handle.c()
    _check("ep_low_latency_dispatch", lib.ep_low_latency_dispatch(
        T, H, K, num_experts, num_max_tokens, x.data_ptr(), topk_idx.data_ptr(),
        recv_x.data_ptr(), recv_scales.data_ptr(), recv_expert_count.data_ptr(), ctypes.byref(c),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_low_latency_combine(expert_out: torch.Tensor, handle: LowLatencyHandle,
                           topk_weights: torch.Tensor, y: torch.Tensor, workspace: torch.Tensor,
                           stream=None) -> None:
    _need(expert_out, "expert_out", torch.bfloat16)
    E, cap, H = expert_out.shape
    T, K = topk_weights.shape
    _need(topk_weights, "topk_weights", torch.float32)
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, K))
    _need(y, "y", torch.bfloat16, shape=(T, H))
    _need(workspace, "workspace", torch.uint8)
    c = handle.c()
    _check("ep_low_latency_combine", lib.ep_low_latency_combine(
        T, H, K, E, cap, expert_out.data_ptr(), ctypes.byref(c), topk_weights.data_ptr(),
        y.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_lb_prefetch_weights(primary_of: torch.Tensor, weights: torch.Tensor,
                           workspace: torch.Tensor, stream=None) -> None:
    """weights: [num_slots, ...] (any dtype, viewed as bytes per slot), updated in place."""
    _need(primary_of, "primary_of", torch.int32)
    S = primary_of.numel()
    _need(weights, "weights", None)
    if weights.shape[0] != S:
        raise ValueError("weights must have one row (blob) per slot")
    nbytes = weights.numel() * weights.element_size() // max(S, 1)
    _need(workspace, "workspace", torch.uint8)
    _check("ep_lb_prefetch_weights", lib.ep_lb_prefetch_weights(
        S, nbytes, primary_of.data_ptr(), weights.data_ptr(), workspace.data_ptr(),
        workspace.numel(), _stream(stream)))


def ep_lb_reduce_grads(primary_of: torch.Tensor, grads: torch.Tensor, workspace: torch.Tensor,
                       stream=None) -> None:
    """grads: float32 [num_slots, n], updated in place."""
    _need(primary_of, "primary_of", torch.int32)
    S = primary_of.numel()
    _need(grads, "grads", torch.float32)
    if grads.shape[0] != S:
        raise ValueError("grads must have one row per slot")
    n = grads.numel() // max(S, 1)
    _need(workspace, "workspace", torch.uint8)
    _check("ep_lb_reduce_grads", lib.ep_lb_reduce_grads(
        S, n, primary_of.data_ptr(), grads.data_ptr(), workspace.data_ptr(), workspace.numel(),
        _stream(stream)))


def ep_debug_wait_probe(timeout_ns: int, workspace: torch.Tensor, stream=None) -> None:
    _need(workspace, "workspace", torch.uint8)
    _check("ep_debug_wait_probe", lib.ep_debug_wait_probe(
        int(timeout_ns), workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_dispatch_backward(grad_recv_x: torch.Tensor, handle: Layout, grad_x: torch.Tensor,
                         workspace: torch.Tensor, grad_recv_topk_weights=None,
                         grad_topk_weights=None, stream=None) -> None:
    _need(grad_recv_x, "grad_recv_x", torch.bfloat16)
    H = grad_recv_x.shape[-1]
    rows = grad_recv_x.numel() // H if H else 0
    T, K = handle.row_of.shape
    _need(handle.row_of, "handle.row_of", torch.int32)
    _need(grad_x, "grad_x", torch.bfloat16, shape=(T, H))
    _need(workspace, "workspace", torch.uint8)
    if grad_recv_topk_weights is not None:
        _need(grad_recv_topk_weights, "grad_recv_topk_weights", torch.float32,
              numel_at_least=rows)
        _need(grad_topk_weights, "grad_topk_weights", torch.float32, shape=(T, K))
    c = ep_layout(row_of=handle.row_of.data_ptr())
    _check("ep_dispatch_backward", lib.ep_dispatch_backward(
        T, H, K, grad_recv_x.data_ptr(), rows, ctypes.byref(c), _ptr(grad_recv_topk_weights),
        grad_x.data_ptr(), _ptr(grad_topk_weights), workspace.data_ptr(), workspace.numel(),
        _stream(stream)))


def ep_combine_backward(grad_y: torch.Tensor, expert_out: torch.Tensor, handle: Layout,
                        topk_weights: torch.Tensor, grad_expert_out: torch.Tensor,
                        grad_topk_weights: torch.Tensor, workspace: torch.Tensor,
                        stream=None) -> None:
    _need(grad_y, "grad_y", torch.bfloat16)
    T, H = grad_y.shape
    _need(expert_out, "expert_out", torch.bfloat16)
    rows = expert_out.numel() // H if H else 0
    K = handle.row_of.shape[1]
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, K))
    _need(topk_weights, "topk_weights", torch.float32, shape=(T, K))
    _need(grad_expert_out, "grad_expert_out", torch.bfloat16, numel_at_least=rows * H)
    _need(grad_topk_weights, "grad_topk_weights", torch.float32, shape=(T, K))
    _need(workspace, "workspace", torch.uint8)
    c = ep_layout(row_of=handle.row_of.data_ptr())
    _check("ep_combine_backward", lib.ep_combine_backward(
        T, H, K, grad_y.data_ptr(), expert_out.data_ptr(), rows, ctypes.byref(c),
        topk_weights.data_ptr(), grad_expert_out.data_ptr(), grad_topk_weights.data_ptr(),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_dispatch_dedup(x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                      num_experts: int, num_partitions: int, quant: int, recv_x: torch.Tensor,
                      recv_scales: Optional[torch.Tensor], recv_topk_idx: torch.Tensor,
                      recv_topk_weights: torch.Tensor, handle: Layout, workspace: torch.Tensor,
                      stream=None) -> None:
    """Deduplicated dispatch; handle = Layout.empty(T, P, P, P) (partition-sized)."""
    _need(x, "x", torch.bfloat16)
    T, H = x.shape
    K = topk_idx.shape[1]
    P = num_partitions
    rows = max(T * min(P, K), 1)
    _need(topk_idx, "topk_idx", torch.int64, shape=(T, K))
    _need(topk_weights, "topk_weights", torch.float32, shape=(T, K))
    if quant & ~EP_QUANT_SCALES_MN_MAJOR in (EP_QUANT_FP8_E4M3_1X128, EP_QUANT_FP8_E4M3_1X128_POW2):
        _need(recv_x, "recv_x", (torch.uint8, torch.float8_e4m3fn), numel_at_least=rows * H)
        _need(recv_scales, "recv_scales", torch.float32,
              numel_at_least=_scale_numel(quant, T * min(P, K), H))
    else:
        _need(recv_x, "recv_x", torch.bfloat16, numel_at_least=rows * H)
    _need(recv_topk_idx, "recv_topk_idx", torch.int32, numel_at_least=rows * K)
    _need(recv_topk_weights, "recv_topk_weights", torch.float32, numel_at_least=rows * K)
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, P))
    _need(handle.src_of, "handle.src_of", torch.int32, numel_at_least=rows)
    _need(handle.num_tokens_per_expert, "handle.num_tokens_per_expert", torch.int32, shape=(P,))
    _need(handle.expert_offset, "handle.expert_offset", torch.int32, shape=(P + 1,))
    _need(handle.is_token_in_partition, "handle.is_token_in_partition", torch.uint8,
          shape=(T, P))
    _need(workspace, "workspace", torch.uint8)
    c = handle.c()
    _check("ep_dispatch_dedup", lib.ep_dispatch_dedup(
        T, H, K, num_experts, P, quant, x.data_ptr(), topk_idx.data_ptr(),
        topk_weights.data_ptr(), recv_x.data_ptr(), _ptr(recv_scales), recv_topk_idx.data_ptr(),
        recv_topk_weights.data_ptr(), ctypes.byref(c), workspace.data_ptr(), workspace.numel(),
        _stream(stream)))


def ep_combine_dedup(partition_out: torch.Tensor, handle: Layout, y: torch.Tensor,
                     workspace: torch.Tensor, stream=None) -> None:
    _need(partition_out, "partition_out", torch.bfloat16)
    H = partition_out.shape[-1]
    rows = partition_out.numel() // H if H else 0
    T, P = handle.row_of.shape
    _need(handle.row_of, "handle.row_of", torch.int32)
    _need(y, "y", torch.bfloat16, shape=(T, H))
    _need(workspace, "workspace", torch.uint8)
    c = ep_layout(row_of=handle.row_of.data_ptr())
    _check("ep_combine_dedup", lib.ep_combine_dedup(
        T, H, P, partition_out.data_ptr(), rows, ctypes.byref(c), y.data_ptr(),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


# ------------------------------------------------ expert parallelism across GPUs --

@dataclass
class PeerTables:
    """Every rank's receive buffers as device tables of W addresses (int64 [W],
    rank order), the ``void* const*`` arguments of ep_peer_dispatch / ep_peer_combine."""

    recv_x: torch.Tensor
    recv_scales: torch.Tensor
    recv_topk_idx: torch.Tensor
    recv_topk_weights: torch.Tensor
    expert_out: torch.Tensor
    capacity: int

    @staticmethod
    def from_addresses(device, capacity: int, recv_x, recv_scales, recv_topk_idx,
                       recv_topk_weights, expert_out) -> "PeerTables":
        def table(addrs):
            return torch.tensor([int(a) for a in addrs], dtype=torch.int64, device=device)
        return PeerTables(table(recv_x), table(recv_scales), table(recv_topk_idx),
                          table(recv_topk_weights), table(expert_out), int(capacity))


class _DeviceMemory:
    """Raw device memory exposed through __cuda_array_interface__ (bytes)."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1",
                                         "data": (ptr, False), "version": 3, "strides": None}


def device_bytes(ptr: int, nbytes: int, device) -> torch.Tensor:
    """A uint8 tensor over `nbytes` of device memory at `ptr` (no copy; the memory
    must outlive the tensor)."""
    return torch.as_tensor(_DeviceMemory(int(ptr), int(nbytes)), device=device)


def ep_ipc_alloc(nbytes: int):
    """Device memory that other processes can map: returns (address, handle bytes)."""
    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(EP_IPC_HANDLE_BYTES)
    _check("ep_ipc_alloc", lib.ep_ipc_alloc(int(nbytes), ctypes.byref(ptr), handle))
    return int(ptr.value), handle.raw


def ep_ipc_free(ptr: int) -> None:
    _check("ep_ipc_free", lib.ep_ipc_free(ptr))


def ep_ipc_open(handle: bytes) -> int:
    if len(handle) != EP_IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {EP_IPC_HANDLE_BYTES} bytes")
    ptr = ctypes.c_void_p()
    _check("ep_ipc_open", lib.ep_ipc_open(handle, ctypes.byref(ptr)))
    return int(ptr.value)


def ep_ipc_close(ptr: int) -> None:
    _check("ep_ipc_close", lib.ep_ipc_close(ptr))


def ep_peer_plan(counts: torch.Tensor, rank: int, expert_offset: torch.Tensor, capacity: int,
                 dst_offset: torch.Tensor, recv_count: torch.Tensor, recv_offset: torch.Tensor,
                 workspace: torch.Tensor, stream=None) -> None:
    """counts: int32 [W, E], every rank's num_tokens_per_expert."""
    _need(counts, "counts", torch.int32)
    W, E = counts.shape
    _need(expert_offset, "expert_offset", torch.int32, shape=(E + 1,))
    _need(dst_offset, "dst_offset", torch.int32, shape=(E,))
    _need(recv_count, "recv_count", torch.int32, shape=(E // W,))
    _need(recv_offset, "recv_offset", torch.int32, shape=(E // W + 1,))
    _need(workspace, "workspace", torch.uint8)
    _check("ep_peer_plan", lib.ep_peer_plan(
        W, rank, E, counts.data_ptr(), expert_offset.data_ptr(), int(capacity),
        dst_offset.data_ptr(), recv_count.data_ptr(), recv_offset.data_ptr(),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_peer_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                     num_experts: int, world: int, quant: int, handle: Layout,
                     dst_offset: torch.Tensor, tables: PeerTables, workspace: torch.Tensor,
                     stream=None) -> None:
    _need(x, "x", torch.bfloat16)
    T, H = x.shape
    K = topk_idx.shape[1]
    _need(topk_idx, "topk_idx", torch.int64, shape=(T, K))
    _need(topk_weights, "topk_weights", torch.float32, shape=(T, K))
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, K))
    _need(dst_offset, "dst_offset", torch.int32, shape=(num_experts,))
    for name in ("recv_x", "recv_scales", "recv_topk_idx", "recv_topk_weights"):
        _need(getattr(tables, name), "tables." + name, torch.int64, shape=(world,))
    _need(workspace, "workspace", torch.uint8)
    c = ep_layout(row_of=handle.row_of.data_ptr())
    fp8 = quant != EP_QUANT_NONE
    b = ep_peer_buffers(tables.recv_x.data_ptr(),
                        tables.recv_scales.data_ptr() if fp8 else None,
                        tables.recv_topk_idx.data_ptr(), tables.recv_topk_weights.data_ptr(),
                        tables.capacity)
    _check("ep_peer_dispatch", lib.ep_peer_dispatch(
        T, H, K, num_experts, world, quant, x.data_ptr(), topk_idx.data_ptr(),
        topk_weights.data_ptr(), ctypes.byref(c), dst_offset.data_ptr(), ctypes.byref(b),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_peer_combine(tables: PeerTables, handle: Layout, topk_idx: torch.Tensor,
                    dst_offset: torch.Tensor, topk_weights: torch.Tensor, y: torch.Tensor,
                    num_experts: int, world: int, workspace: torch.Tensor, stream=None) -> None:
    _need(y, "y", torch.bfloat16)
    T, H = y.shape
    K = topk_idx.shape[1]
    _need(topk_idx, "topk_idx", torch.int64, shape=(T, K))
    _need(topk_weights, "topk_weights", torch.float32, shape=(T, K))
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, K))
    _need(dst_offset, "dst_offset", torch.int32, shape=(num_experts,))
    _need(tables.expert_out, "tables.expert_out", torch.int64, shape=(world,))
    _need(workspace, "workspace", torch.uint8)
    c = ep_layout(row_of=handle.row_of.data_ptr())
    _check("ep_peer_combine", lib.ep_peer_combine(
        T, H, K, num_experts, world, tables.expert_out.data_ptr(), tables.capacity,
        ctypes.byref(c), topk_idx.data_ptr(), dst_offset.data_ptr(), topk_weights.data_ptr(),
        y.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_get_dispatch_layout_dedup(topk_idx: torch.Tensor, num_experts: int, num_partitions: int,
                                 layout: Layout, workspace: torch.Tensor, stream=None) -> None:
    """The deduplicated layout; layout = Layout.empty(T, P, P, P) (partition-sized)."""
    _need(topk_idx, "topk_idx", torch.int64)
    T, K = topk_idx.shape
    P = num_partitions
    _need(layout.row_of, "layout.row_of", torch.int32, shape=(T, P))
    _need(layout.num_tokens_per_expert, "layout.num_tokens_per_expert", torch.int32, shape=(P,))
    _need(layout.num_tokens_per_partition, "layout.num_tokens_per_partition", torch.int32,
          shape=(P,))
    _need(layout.is_token_in_partition, "layout.is_token_in_partition", torch.uint8, shape=(T, P))
    _need(layout.expert_offset, "layout.expert_offset", torch.int32, shape=(P + 1,))
    _need(layout.src_of, "layout.src_of", torch.int32, numel_at_least=T * min(P, K))
    _need(workspace, "workspace", torch.uint8)
    c = layout.c()
    _check("ep_get_dispatch_layout_dedup", lib.ep_get_dispatch_layout_dedup(
        T, K, num_experts, P, topk_idx.data_ptr(), ctypes.byref(c), workspace.data_ptr(),
        workspace.numel(), _stream(stream)))


def ep_peer_dispatch_dedup(x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                           num_experts: int, world: int, quant: int, handle: Layout,
                           dst_offset: torch.Tensor, tables: PeerTables, workspace: torch.Tensor,
                           stream=None) -> None:
    """Rows per (token, rank); the id / weight tables point to [capacity, K] arrays."""
    _need(x, "x", torch.bfloat16)
    T, H = x.shape
    K = topk_idx.shape[1]
    _need(topk_idx, "topk_idx", torch.int64, shape=(T, K))
    _need(topk_weights, "topk_weights", torch.float32, shape=(T, K))
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, world))
    _need(dst_offset, "dst_offset", torch.int32, shape=(world,))
    for name in ("recv_x", "recv_scales", "recv_topk_idx", "recv_topk_weights"):
        _need(getattr(tables, name), "tables." + name, torch.int64, shape=(world,))
    _need(workspace, "workspace", torch.uint8)
    c = ep_layout(row_of=handle.row_of.data_ptr())
    fp8 = quant != EP_QUANT_NONE
    b = ep_peer_buffers(tables.recv_x.data_ptr(),
                        tables.recv_scales.data_ptr() if fp8 else None,
                        tables.recv_topk_idx.data_ptr(), tables.recv_topk_weights.data_ptr(),
                        tables.capacity)
    _check("ep_peer_dispatch_dedup", lib.ep_peer_dispatch_dedup(
        T, H, K, num_experts, world, quant, x.data_ptr(), topk_idx.data_ptr(),
        topk_weights.data_ptr(), ctypes.byref(c), dst_offset.data_ptr(), ctypes.byref(b),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_peer_combine_dedup(tables: PeerTables, handle: Layout, dst_offset: torch.Tensor,
                          y: torch.Tensor, world: int, workspace: torch.Tensor,
                          stream=None) -> None:
    """y[t] = sum over ranks q (in order) of rank q's partition output for (t, q);
    the outputs are read through tables.expert_out."""
    _need(y, "y", torch.bfloat16)
    T, H = y.shape
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, world))
    _need(dst_offset, "dst_offset", torch.int32, shape=(world,))
    _need(tables.expert_out, "tables.expert_out", torch.int64, shape=(world,))
    _need(workspace, "workspace", torch.uint8)
    c = ep_layout(row_of=handle.row_of.data_ptr())
    _check("ep_peer_combine_dedup", lib.ep_peer_combine_dedup(
        T, H, world, tables.expert_out.data_ptr(), tables.capacity, ctypes.byref(c),
        dst_offset.data_ptr(), y.data_ptr(), workspace.data_ptr(), workspace.numel(),
        _stream(stream)))


def ep_peer_low_latency_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, num_max_tokens: int,
                                 num_experts: int, world: int, rank: int, recv_x: torch.Tensor,
                                 recv_scales: torch.Tensor, recv_expert_count: torch.Tensor,
                                 handle: LowLatencyHandle, workspace: torch.Tensor,
                                 stream=None) -> None:
    """recv_x / recv_scales / recv_expert_count: int64 [W] device tables of every rank's
    [E/W, W*cap, H] E4M3, [E/W, W*cap, H/128] fp32 and [E/W, W] int32 buffers."""
    _need(x, "x", torch.bfloat16)
    T, H = x.shape
    K = topk_idx.shape[1]
    _need(topk_idx, "topk_idx", torch.int64, shape=(T, K))
    for name, t in (("recv_x", recv_x), ("recv_scales", recv_scales),
                    ("recv_expert_count", recv_expert_count)):
        _need(t, name, torch.int64, shape=(world,))
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, K))
    _need(handle.src_of, "handle.src_of", torch.int32, shape=(num_experts, num_max_tokens))
    _need(workspace, "workspace", torch.uint8)
    c = handle.c()
    _check("ep_peer_low_latency_dispatch", lib.ep_peer_low_latency_dispatch(
        T, H, K, num_experts, world, rank, num_max_tokens, x.data_ptr(), topk_idx.data_ptr(),
        recv_x.data_ptr(), recv_scales.data_ptr(), recv_expert_count.data_ptr(), ctypes.byref(c),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def ep_peer_low_latency_combine(expert_out: torch.Tensor, topk_idx: torch.Tensor,
                                handle: LowLatencyHandle, topk_weights: torch.Tensor,
                                y: torch.Tensor, num_experts: int, world: int, rank: int,
                                workspace: torch.Tensor, stream=None) -> None:
    """expert_out: int64 [W] device table of every rank's BF16 [E/W, W*cap, H] outputs."""
    _need(y, "y", torch.bfloat16)
    T, H = y.shape
    K = topk_idx.shape[1]
    _need(topk_idx, "topk_idx", torch.int64, shape=(T, K))
    _need(topk_weights, "topk_weights", torch.float32, shape=(T, K))
    _need(expert_out, "expert_out", torch.int64, shape=(world,))
    _need(handle.row_of, "handle.row_of", torch.int32, shape=(T, K))
    _need(workspace, "workspace", torch.uint8)
    c = handle.c()
    _check("ep_peer_low_latency_combine", lib.ep_peer_low_latency_combine(
        T, H, K, num_experts, world, rank, handle.num_max_tokens, expert_out.data_ptr(),
        topk_idx.data_ptr(), ctypes.byref(c), topk_weights.data_ptr(), y.data_ptr(),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))
