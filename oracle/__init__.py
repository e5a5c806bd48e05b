"""CPU oracle for MoE token dispatch / combine -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.

This module is argument marshalling (numpy <-> ctypes) around the plain C
statement in ``ep_oracle.c``; every arithmetic step lives there, with the
passage of the DeepEP pages it follows.  Status bits returned by the C
functions: 1 = an index outside its range was skipped, 4 = a low-latency row
did not fit its expert's capacity.
"""
from __future__ import annotations

import ctypes
from typing import Dict

import numpy as np

from . import build as _build

INDEX_RANGE = 1
CAPACITY = 4

_lib = None

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_p = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_bf16_from_f32.argtypes = [ctypes.c_float]
        L.oracle_bf16_from_f32.restype = ctypes.c_uint16
        L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_f32.restype = ctypes.c_float
        L.oracle_e4m3_from_f32.argtypes = [ctypes.c_float]
        L.oracle_e4m3_from_f32.restype = ctypes.c_uint8
        L.oracle_e4m3_from_f32_n.argtypes = [_i64, _p, _p]
        L.oracle_e4m3_from_f32_n.restype = None
        L.oracle_bf16_from_f32_n.argtypes = [_i64, _p, _p]
        L.oracle_bf16_from_f32_n.restype = None
        L.oracle_block_scale.argtypes = [ctypes.c_float]
        L.oracle_block_scale.restype = ctypes.c_float
        L.oracle_block_scale_pow2.argtypes = [ctypes.c_float]
        L.oracle_block_scale_pow2.restype = ctypes.c_float
        L.oracle_quantize_row_mode.argtypes = [_i64, _p, _p, _p, _i32]
        L.oracle_quantize_row_mode.restype = None
        L.oracle_quantize_row.argtypes = [_i64, _p, _p, _p]
        L.oracle_quantize_row.restype = None
        L.oracle_layout.argtypes = [_i64, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p, _p, _p]
        L.oracle_layout.restype = ctypes.c_uint32
        L.oracle_dispatch.argtypes = [_i64, _i64, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p,
                                      _p, _p]
        L.oracle_dispatch.restype = ctypes.c_uint32
        L.oracle_identity_expert.argtypes = [_i64, _i64, _i32, _p, _p, _p]
        L.oracle_identity_expert.restype = None
        L.oracle_combine.argtypes = [_i64, _i64, _i32, _p, _i64, _p, _p, _p]
        L.oracle_combine.restype = ctypes.c_uint32
        L.oracle_ll_dispatch.argtypes = [_i64, _i64, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p, _p]
        L.oracle_ll_dispatch.restype = ctypes.c_uint32
        L.oracle_dispatch_backward.argtypes = [_i64, _i64, _i32, _p, _i64, _p, _p, _p, _p]
        L.oracle_dispatch_backward.restype = ctypes.c_uint32
        L.oracle_combine_backward.argtypes = [_i64, _i64, _i32, _p, _p, _i64, _p, _p, _p, _p]
        L.oracle_combine_backward.restype = ctypes.c_uint32
        L.oracle_dispatch_dedup.argtypes = [_i64, _i64, _i32, _i32, _i32, _i32, _p, _p, _p, _p,
                                            _p, _p, _p, _p, _p, _p, _p, _p]
        L.oracle_dispatch_dedup.restype = ctypes.c_uint32
        L.oracle_partition_identity.argtypes = [_i64, _i64, _i32, _i32, _p, _p, _p, _p, _p]
        L.oracle_partition_identity.restype = None
        L.oracle_combine_dedup.argtypes = [_i64, _i64, _i32, _p, _i64, _p, _p]
        L.oracle_lb_prefetch_weights.argtypes = [_i32, _i64, _p, _p]
        L.oracle_lb_prefetch_weights.restype = ctypes.c_uint32
        L.oracle_lb_reduce_grads.argtypes = [_i32, _i64, _p, _p]
        L.oracle_lb_reduce_grads.restype = ctypes.c_uint32
        L.oracle_combine_dedup.restype = ctypes.c_uint32
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------ scalar codecs --

def bf16_to_f32(b: int) -> float:
    return float(lib().oracle_bf16_to_f32(int(b)))


def bf16_from_f32(v: float) -> int:
    return int(lib().oracle_bf16_from_f32(float(v)))


def e4m3_to_f32(c: int) -> float:
    return float(lib().oracle_e4m3_to_f32(int(c)))


def e4m3_from_f32(v: float) -> int:
    return int(lib().oracle_e4m3_from_f32(float(v)))


def block_scale(amax: float) -> float:
    return float(lib().oracle_block_scale(float(amax)))


def block_scale_pow2(amax: float) -> float:
    return float(lib().oracle_block_scale_pow2(float(amax)))


QUANT_MODES = {"none": 0, "fp8": 1, "fp8_pow2": 2}


# ----------------------------------------------------- vectorised wrappers --
# The array codecs loop in C over the elements; the Python side only moves
# buffers.

def e4m3_from_f32_array(v: np.ndarray) -> np.ndarray:
    """E4M3 codes of a float32 array (elementwise ``oracle_e4m3_from_f32``)."""
    v = _c(v, np.float32).reshape(-1)
    out = np.empty(v.size, dtype=np.uint8)
    if v.size:
        lib().oracle_e4m3_from_f32_n(v.size, _ptr(v), _ptr(out))
    return out


def bf16_from_f32_array(v: np.ndarray) -> np.ndarray:
    """BF16 bit patterns of a float32 array (elementwise ``oracle_bf16_from_f32``)."""
    v = _c(v, np.float32).reshape(-1)
    out = np.empty(v.size, dtype=np.uint16)
    if v.size:
        lib().oracle_bf16_from_f32_n(v.size, _ptr(v), _ptr(out))
    return out


def quantize_row(x_row: np.ndarray, pow2: bool = False):
    """E4M3 codes and 1x128 fp32 scales of one BF16 row (uint16 bit patterns)."""
    x_row = _c(x_row, np.uint16).reshape(-1)
    H = x_row.size
    q = np.empty(H, dtype=np.uint8)
    s = np.empty(H // 128, dtype=np.float32)
    lib().oracle_quantize_row_mode(H, _ptr(x_row), _ptr(q), _ptr(s), 1 if pow2 else 0)
    return q, s


def quantize_rows(x: np.ndarray):
    """Row-wise quantisation of a [T, H] BF16 array."""
    x = _c(x, np.uint16)
    T, H = x.shape
    q = np.empty((T, H), dtype=np.uint8)
    s = np.empty((T, H // 128), dtype=np.float32)
    for t in range(T):
        lib().oracle_quantize_row(H, _ptr(x[t]), _ptr(q[t]), _ptr(s[t]))
    return q, s


# ------------------------------------------------------------------ layout --

def layout(topk_idx: np.ndarray, num_experts: int, num_partitions: int) -> Dict[str, np.ndarray]:
    idx = _c(topk_idx, np.int64)
    T, K = idx.shape
    E, P = num_experts, num_partitions
    out = dict(
        num_tokens_per_expert=np.empty(E, np.int32),
        num_tokens_per_partition=np.empty(P, np.int32),
        is_token_in_partition=np.empty((T, P), np.uint8),
        expert_offset=np.empty(E + 1, np.int32),
        row_of=np.empty((T, K), np.int32),
        src_of=np.full(max(T * K, 1), -1, np.int32),
        num_recv=np.zeros(1, np.int32),
    )
    st = lib().oracle_layout(T, K, E, P, _ptr(idx), _ptr(out["num_tokens_per_expert"]),
                             _ptr(out["num_tokens_per_partition"]),
                             _ptr(out["is_token_in_partition"]), _ptr(out["expert_offset"]),
                             _ptr(out["row_of"]), _ptr(out["src_of"]), _ptr(out["num_recv"]))
    out["src_of"] = out["src_of"][: int(out["num_recv"][0])].copy()
    out["status"] = int(st)
    return out


# ---------------------------------------------------------------- dispatch --

def dispatch(x: np.ndarray, topk_idx: np.ndarray, topk_weights: np.ndarray, num_experts: int,
             num_partitions: int, quant: str = "fp8") -> Dict[str, np.ndarray]:
    """Layout + dispatch.  Returns the layout dict plus recv_x / recv_scales /
    recv_topk_idx / recv_topk_weights with exactly num_recv rows."""
    x = _c(x, np.uint16)
    idx = _c(topk_idx, np.int64)
    w = _c(topk_weights, np.float32)
    T, H = x.shape
    K = idx.shape[1]
    lay = layout(idx, num_experts, num_partitions)
    R = int(lay["num_recv"][0])
    qm = QUANT_MODES[quant]
    rows = max(R, 1)
    recv_x = np.zeros((rows, H), np.uint8) if qm else np.zeros((rows, H), np.uint16)
    recv_scales = np.zeros((rows, max(H // 128, 1)), np.float32)
    recv_topk_idx = np.zeros(rows, np.int32)
    recv_topk_weights = np.zeros(rows, np.float32)
    st = lib().oracle_dispatch(T, H, K, num_experts, num_partitions, qm, _ptr(x), _ptr(idx),
                               _ptr(w), _ptr(lay["row_of"]), _ptr(recv_x), _ptr(recv_scales),
                               _ptr(recv_topk_idx), _ptr(recv_topk_weights))
    lay.update(recv_x=recv_x[:R], recv_scales=recv_scales[:R, : H // 128],
               recv_topk_idx=recv_topk_idx[:R], recv_topk_weights=recv_topk_weights[:R])
    lay["status"] |= int(st)
    return lay


def identity_expert(recv_x: np.ndarray, recv_scales, quant: str = "fp8") -> np.ndarray:
    """BF16 expert output of the identity expert (dequantised receive rows)."""
    R, H = recv_x.shape
    qm = QUANT_MODES[quant]
    rx = _c(recv_x, np.uint8 if qm else np.uint16)
    rs = _c(recv_scales if recv_scales is not None else np.zeros((R, 1), np.float32), np.float32)
    out = np.empty((R, H), np.uint16)
    if R:
        lib().oracle_identity_expert(R, H, qm, _ptr(rx), _ptr(rs), _ptr(out))
    return out


# ----------------------------------------------------------------- combine --

def combine(expert_out: np.ndarray, row_of: np.ndarray, topk_weights: np.ndarray):
    """Weighted k-way gather-reduce back to token order; returns (y, status)."""
    eo = _c(expert_out, np.uint16)
    rows, H = eo.shape
    ro = _c(row_of, np.int32)
    w = _c(topk_weights, np.float32)
    T, K = ro.shape
    y = np.empty((T, H), np.uint16)
    eo_p = eo if rows else np.zeros((1, H), np.uint16)
    st = lib().oracle_combine(T, H, K, _ptr(eo_p), rows, _ptr(ro), _ptr(w), _ptr(y))
    return y, int(st)


# ------------------------------------------------------------- low latency --

def ll_dispatch(x: np.ndarray, topk_idx: np.ndarray, num_experts: int, num_max_tokens: int,
                fill: int = 0xA5) -> Dict[str, np.ndarray]:
    """Padded low-latency dispatch.  Unwritten slots keep ``fill`` (payload bytes)
    / NaN-free sentinel patterns so tests can tell them apart."""
    x = _c(x, np.uint16)
    idx = _c(topk_idx, np.int64)
    T, H = x.shape
    K = idx.shape[1]
    E, cap = num_experts, num_max_tokens
    recv_x = np.full((E, cap, H), fill, np.uint8)
    recv_scales = np.full((E, cap, H // 128), -1.0, np.float32)
    count = np.empty(E, np.int32)
    row_of = np.empty((T, K), np.int32)
    src_of = np.full((E, cap), -1, np.int32)
    st = lib().oracle_ll_dispatch(T, H, K, E, cap, _ptr(x), _ptr(idx), _ptr(recv_x),
                                  _ptr(recv_scales), _ptr(count), _ptr(row_of), _ptr(src_of))
    return dict(recv_x=recv_x, recv_scales=recv_scales, recv_expert_count=count,
                ll_row_of=row_of, ll_src_of=src_of, status=int(st))


def ll_combine(expert_out: np.ndarray, ll_row_of: np.ndarray, topk_weights: np.ndarray):
    """Low-latency combine: the same k-way reduce over a padded [E, cap, H] output."""
    E, cap, H = expert_out.shape
    return combine(expert_out.reshape(E * cap, H), ll_row_of, topk_weights)


# ---------------------------------------------------------------- backward --

def dispatch_backward(grad_recv_x: np.ndarray, row_of: np.ndarray,
                      grad_recv_topk_weights=None):
    """grad_x (BF16 bits [T, H]) and grad_topk_weights (fp32 [T, K] or None)."""
    g = _c(grad_recv_x, np.uint16)
    rows, H = g.shape
    ro = _c(row_of, np.int32)
    T, K = ro.shape
    gx = np.empty((T, H), np.uint16)
    gw = np.zeros((T, K), np.float32) if grad_recv_topk_weights is not None else None
    grw = _c(grad_recv_topk_weights, np.float32) if grad_recv_topk_weights is not None else None
    g_p = g if rows else np.zeros((1, H), np.uint16)
    st = lib().oracle_dispatch_backward(T, H, K, _ptr(g_p), rows, _ptr(ro),
                                        _ptr(grw) if grw is not None else None, _ptr(gx),
                                        _ptr(gw) if gw is not None else None)
    return gx, gw, int(st)


def combine_backward(grad_y: np.ndarray, expert_out: np.ndarray, row_of: np.ndarray,
                     topk_weights: np.ndarray, fill: int = 0xA5A5):
    """grad_expert_out (BF16 bits [rows, H]; rows no slot points at keep `fill`) and
    grad_topk_weights (fp32 [T, K])."""
    gy = _c(grad_y, np.uint16)
    eo = _c(expert_out, np.uint16)
    rows, H = eo.shape
    ro = _c(row_of, np.int32)
    w = _c(topk_weights, np.float32)
    T, K = ro.shape
    geo = np.full((max(rows, 1), H), fill, np.uint16)
    gw = np.empty((T, K), np.float32)
    eo_p = eo if rows else np.zeros((1, H), np.uint16)
    st = lib().oracle_combine_backward(T, H, K, _ptr(gy), _ptr(eo_p), rows, _ptr(ro), _ptr(w),
                                       _ptr(geo), _ptr(gw))
    return geo[:rows], gw, int(st)


# ---------------------------------------------------- deduplicated dispatch --

def dispatch_dedup(x: np.ndarray, topk_idx: np.ndarray, topk_weights: np.ndarray,
                   num_experts: int, num_partitions: int, quant: str = "fp8"):
    """One row per (token, partition).  Returns prow_of [T, P], part_count [P],
    part_offset [P+1], src_tok [rows], num_rows, recv_x, recv_scales,
    recv_topk_idx [rows, K], recv_topk_weights [rows, K], status."""
    x = _c(x, np.uint16)
    idx = _c(topk_idx, np.int64)
    w = _c(topk_weights, np.float32)
    T, H = x.shape
    K = idx.shape[1]
    P = num_partitions
    qm = QUANT_MODES[quant]
    cap = max(T * min(P, K), 1)
    out = dict(prow_of=np.empty((T, P), np.int32), part_count=np.empty(P, np.int32),
               part_offset=np.empty(P + 1, np.int32), src_tok=np.full(cap, -1, np.int32),
               num_rows=np.zeros(1, np.int32),
               recv_x=np.zeros((cap, H), np.uint8 if qm else np.uint16),
               recv_scales=np.zeros((cap, max(H // 128, 1)), np.float32),
               recv_topk_idx=np.zeros((cap, K), np.int32),
               recv_topk_weights=np.zeros((cap, K), np.float32))
    st = lib().oracle_dispatch_dedup(
        T, H, K, num_experts, P, qm, _ptr(x), _ptr(idx), _ptr(w), _ptr(out["prow_of"]),
        _ptr(out["part_count"]), _ptr(out["part_offset"]), _ptr(out["src_tok"]),
        _ptr(out["num_rows"]), _ptr(out["recv_x"]), _ptr(out["recv_scales"]),
        _ptr(out["recv_topk_idx"]), _ptr(out["recv_topk_weights"]))
    R = int(out["num_rows"][0])
    for k in ("src_tok", "recv_x", "recv_topk_idx", "recv_topk_weights"):
        out[k] = out[k][:R]
    out["recv_scales"] = out["recv_scales"][:R, : H // 128]
    out["status"] = int(st)
    return out


def partition_identity(recv_x, recv_scales, recv_topk_idx, recv_topk_weights, quant="fp8"):
    """Partition-local stand-in expert output for the deduplicated path."""
    R, H = recv_x.shape
    K = recv_topk_idx.shape[1]
    qm = 1 if quant == "fp8" else 0
    rx = _c(recv_x, np.uint8 if qm else np.uint16)
    rs = _c(recv_scales if recv_scales is not None else np.zeros((R, 1), np.float32), np.float32)
    ri = _c(recv_topk_idx, np.int32)
    rw = _c(recv_topk_weights, np.float32)
    out = np.empty((R, H), np.uint16)
    if R:
        lib().oracle_partition_identity(R, H, K, qm, _ptr(rx), _ptr(rs), _ptr(ri), _ptr(rw),
                                        _ptr(out))
    return out


def combine_dedup(part_out: np.ndarray, prow_of: np.ndarray):
    po = _c(part_out, np.uint16)
    rows, H = po.shape
    pr = _c(prow_of, np.int32)
    T, P = pr.shape
    y = np.empty((T, H), np.uint16)
    po_p = po if rows else np.zeros((1, H), np.uint16)
    st = lib().oracle_combine_dedup(T, H, P, _ptr(po_p), rows, _ptr(pr), _ptr(y))
    return y, int(st)


def lb_prefetch_weights(weights: np.ndarray, primary_of: np.ndarray):
    """weights: uint8 [S, nbytes] (a copy is returned); primary_of: int32 [S]."""
    w = np.array(weights, dtype=np.uint8, order="C", copy=True)
    S, nbytes = w.shape
    po = _c(primary_of, np.int32)
    st = lib().oracle_lb_prefetch_weights(S, nbytes, _ptr(po), _ptr(w))
    return w, int(st)


def lb_reduce_grads(grads: np.ndarray, primary_of: np.ndarray):
    """grads: float32 [S, n] (a copy is returned); primary_of: int32 [S]."""
    g = np.array(grads, dtype=np.float32, order="C", copy=True)
    S, n = g.shape
    po = _c(primary_of, np.int32)
    st = lib().oracle_lb_reduce_grads(S, n, _ptr(po), _ptr(g))
    return g, int(st)
