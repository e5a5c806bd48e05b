"""DeepEP-style ``Buffer`` on top of the C ABI.

Shapes of the calls follow the DeepEP pages:

* deepseek.csdn.net/67bd3eb22e30c863900615cc, section "使用示例 / MoE 训练中的应用":
  ``recv_x, recv_topk_idx, recv_topk_weights, handle, event =
  buffer.dispatch(x, topk_idx, topk_weights, num_experts)``;
* same page, section "推理解码阶段的应用":
  ``recv_hidden_states, recv_expert_count, handle, event, hook =
  buffer.low_latency_dispatch(hidden_states, topk_idx, num_max_tokens, num_experts)``
  with a buffer of ``num_max_tokens * hidden * num_experts`` elements;
* "deepseek-ai/DeepEP" (agentlenshq.com), section "典型工作流程": dispatch, expert
  GEMM, ``buffer.combine(...)`` (or the backward helpers) reduces the expert
  outputs back.

Besides the per-expert dispatch (one receive row per token and expert), the
buffer offers the deduplicated dispatch (one row per token and partition, with
the partition's expert list per row) and the backward pair.

Everything runs on one GPU: the ``num_partitions`` logical partitions stand for
the EP ranks, so there is no process group.  torch provides device memory and
the stream; every step runs in the library's kernels.  ``event`` is a
``torch.cuda.Event`` recorded after the launches.  The low-latency ``hook`` is
a no-op callable: on one GPU there is no receive phase to defer.
"""
from __future__ import annotations

from typing import Optional, Union

import torch

from . import _lib
from ._lib import (EP_QUANT_FP8_E4M3_1X128, EP_QUANT_FP8_E4M3_1X128_POW2, EP_QUANT_NONE,
                   EP_QUANT_SCALES_MN_MAJOR, Layout, LowLatencyHandle, scales_ld)

__all__ = ["Buffer"]


def _noop_hook():
    return None


class Buffer:
    """Dispatch / combine buffer for one GPU.

    Call shapes: ``Buffer(group, num_nvl_bytes, num_rdma_bytes[, low_latency_mode])``
    as on the pages (deepseek.csdn.net/67bd3eb22e30c863900615cc, sections
    "使用示例" and "推理解码阶段的应用"), or by keyword ``Buffer(num_experts=,
    num_partitions=, max_tokens=)``.

    ``num_partitions`` logical partitions (the EP ranks of a multi-GPU run) split
    the experts into equal contiguous ranges; it defaults to ``group.size()`` when
    a process group is given, else 1.  ``num_nvl_bytes`` / ``num_rdma_bytes`` size
    DeepEP's peer buffers; one GPU has none, so they are recorded and unused.
    ``low_latency_mode`` is recorded; both kinds of calls are always available.
    ``num_experts`` may be left to the first call that passes it.  The device
    workspace is sized for the largest batch seen so far (``max_tokens`` to start)
    and grows, on the current stream, when a larger batch arrives.
    """

    def __init__(self, group=None, num_nvl_bytes: int = 0, num_rdma_bytes: int = 0,
                 low_latency_mode: bool = False, *, num_experts: Optional[int] = None,
                 num_partitions: Optional[int] = None, max_tokens: int = 0,
                 device: Optional[Union[int, str, torch.device]] = None):
        if num_partitions is None:
            num_partitions = group.size() if group is not None else 1
        if num_experts is not None and num_experts % num_partitions:
            raise ValueError("num_experts must be a multiple of num_partitions")
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.group = group
        self.num_nvl_bytes = num_nvl_bytes
        self.num_rdma_bytes = num_rdma_bytes
        self.low_latency_mode = low_latency_mode
        self.num_experts = num_experts
        self.num_partitions = num_partitions
        self.max_tokens = max_tokens
        self.workspace: Optional[torch.Tensor] = None
        self._ensure(max_tokens)

    # ------------------------------------------------------------ helpers --
    def _ensure(self, num_tokens: int, num_experts: Optional[int] = None) -> None:
        """Fix num_experts on first use and grow the workspace to fit the batch."""
        if num_experts is not None:
            if self.num_experts is None:
                if num_experts % self.num_partitions:
                    raise ValueError("num_experts must be a multiple of num_partitions")
                self.num_experts = num_experts
                self.workspace = None  # sized for the experts now known
            elif num_experts != self.num_experts:
                raise ValueError("num_experts differs from the buffer's")
        self.max_tokens = max(self.max_tokens, num_tokens)
        need = _lib.ep_workspace_bytes(max(self.max_tokens, 1), self.num_experts or 1,
                                       self.num_partitions)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
            _lib.ep_workspace_init(self.workspace)

    def _experts(self) -> int:
        if self.num_experts is None:
            raise ValueError("num_experts is not known yet: pass it to this call or to Buffer()")
        return self.num_experts

    def _event(self) -> torch.cuda.Event:
        ev = torch.cuda.Event()
        ev.record()
        return ev

    def read_status(self) -> int:
        """Synchronise and return (then clear) the sticky device status bits."""
        return _lib.ep_read_status(self.workspace)

    # ------------------------------------------------------------- layout --
    def get_dispatch_layout(self, topk_idx: torch.Tensor):
        """Returns ``(num_tokens_per_expert, num_tokens_per_partition,
        is_token_in_partition, handle, event)``."""
        T, K = topk_idx.shape
        self._ensure(T)
        E = self._experts()
        lay = Layout.empty(T, K, E, self.num_partitions, self.device)
        _lib.ep_get_dispatch_layout(topk_idx, E, self.num_partitions, lay,
                                    self.workspace)
        return (lay.num_tokens_per_expert, lay.num_tokens_per_partition,
                lay.is_token_in_partition, lay, self._event())

    # ----------------------------------------------------------- dispatch --
    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                 num_experts: Optional[int] = None, use_fp8: bool = True, exact: bool = True,
                 pow2_scales: bool = False, scales_mn_major: bool = False):
        """Returns ``(recv_x, recv_topk_idx, recv_topk_weights, handle, event)``.

        With ``use_fp8`` recv_x is ``(payload float8_e4m3fn [R, H], scales float32
        [R, H/128])``; otherwise a BF16 ``[R, H]`` tensor.  ``pow2_scales`` rounds
        every scale up to a power of two; ``scales_mn_major`` stores the scales
        block-major (the [R, H/128] tensor is then a strided view of an
        [H/128, ld] buffer, the layout FP8 grouped GEMMs read).  ``exact`` trims the
        worst-case (T*K-row) buffers to the R received rows, which reads R back to
        the host once; ``exact=False`` returns the untrimmed buffers and never
        synchronises (R is then ``handle.num_recv`` on the device).
        """
        T, H = x.shape
        K = topk_idx.shape[1]
        self._ensure(T, num_experts)
        self._experts()
        rows = max(T * K, 1)
        dev = self.device
        handle = Layout.empty(T, K, self.num_experts, self.num_partitions, dev)
        recv_topk_idx = torch.empty(rows, dtype=torch.int32, device=dev)
        recv_topk_weights = torch.empty(rows, dtype=torch.float32, device=dev)
        if use_fp8:
            recv_q = torch.empty((rows, H), dtype=torch.float8_e4m3fn, device=dev)
            quant = EP_QUANT_FP8_E4M3_1X128_POW2 if pow2_scales else EP_QUANT_FP8_E4M3_1X128
            if scales_mn_major:
                quant |= EP_QUANT_SCALES_MN_MAJOR
                flat = torch.empty((H // 128, scales_ld(rows)), dtype=torch.float32, device=dev)
                recv_s = flat.t()[:rows]
            else:
                flat = recv_s = torch.empty((rows, H // 128), dtype=torch.float32, device=dev)
            _lib.ep_dispatch(x, topk_idx, topk_weights, self.num_experts, self.num_partitions,
                             quant, recv_q, flat, recv_topk_idx, recv_topk_weights, handle,
                             self.workspace)
        else:
            recv_q = torch.empty((rows, H), dtype=torch.bfloat16, device=dev)
            recv_s = None
            _lib.ep_dispatch(x, topk_idx, topk_weights, self.num_experts, self.num_partitions,
                             EP_QUANT_NONE, recv_q, None, recv_topk_idx, recv_topk_weights,
                             handle, self.workspace)
        event = self._event()
        if exact:
            R = int(handle.num_recv.item())
            recv_q, recv_topk_idx, recv_topk_weights = recv_q[:R], recv_topk_idx[:R], \
                recv_topk_weights[:R]
            if recv_s is not None:
                recv_s = recv_s[:R]
        recv_x = (recv_q, recv_s) if use_fp8 else recv_q
        return recv_x, recv_topk_idx, recv_topk_weights, handle, event

    # ------------------------------------------------------------ combine --
    def combine(self, expert_out: torch.Tensor, handle: Layout, topk_weights: torch.Tensor):
        """Returns ``(y, event)``: y[t] = bf16(sum_k w[t,k] * expert_out[row_of[t,k]])."""
        T = topk_weights.shape[0]
        H = expert_out.shape[-1]
        y = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)
        _lib.ep_combine(expert_out, handle, topk_weights, y, self.workspace)
        return y, self._event()

    # -------------------------------------------------------- low latency --
    def low_latency_dispatch(self, hidden_states: torch.Tensor, topk_idx: torch.Tensor,
                             num_max_tokens: int, num_experts: Optional[int] = None):
        """Returns ``(recv_hidden_states, recv_expert_count, handle, event, hook)``.

        recv_hidden_states is ``(payload float8_e4m3fn [E, num_max_tokens, H],
        scales float32 [E, num_max_tokens, H/128])``; slots at or beyond
        recv_expert_count[e] are not written.
        """
        E = self.num_experts if num_experts is None else num_experts
        if E is None:
            raise ValueError("num_experts is not known yet: pass it to this call or to Buffer()")
        T, H = hidden_states.shape
        K = topk_idx.shape[1]
        dev = self.device
        recv_q = torch.empty((E, num_max_tokens, H), dtype=torch.float8_e4m3fn, device=dev)
        recv_s = torch.empty((E, num_max_tokens, H // 128), dtype=torch.float32, device=dev)
        count = torch.empty(E, dtype=torch.int32, device=dev)
        handle = LowLatencyHandle.empty(T, K, E, num_max_tokens, dev)
        _lib.ep_low_latency_dispatch(hidden_states, topk_idx, num_max_tokens, E, recv_q, recv_s,
                                     count, handle, self.workspace)
        return (recv_q, recv_s), count, handle, self._event(), _noop_hook

    def low_latency_combine(self, expert_out: torch.Tensor, topk_idx: Optional[torch.Tensor],
                            topk_weights: torch.Tensor, handle: LowLatencyHandle):
        """Returns ``(y, event, hook)``.  ``topk_idx`` is accepted for call-shape
        compatibility; the rows come from the handle."""
        T = topk_weights.shape[0]
        H = expert_out.shape[-1]
        y = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)
        _lib.ep_low_latency_combine(expert_out, handle, topk_weights, y, self.workspace)
        return y, self._event(), _noop_hook

    # ------------------------------------------------------- deduplicated --
    def dispatch_dedup(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                       use_fp8: bool = True, exact: bool = True, pow2_scales: bool = False):
        """One receive row per (token, partition).  Returns ``(recv_x, recv_topk_idx
        [R, K], recv_topk_weights [R, K], handle, event)``; handle.row_of is [T, P]."""
        T, H = x.shape
        K = topk_idx.shape[1]
        P = self.num_partitions
        self._ensure(T)
        self._experts()
        if P > 32:
            raise ValueError("the deduplicated dispatch supports at most 32 partitions")
        rows = max(T * min(P, K), 1)
        dev = self.device
        handle = Layout.empty(T, P, P, P, dev)
        ri = torch.empty((rows, K), dtype=torch.int32, device=dev)
        rw = torch.empty((rows, K), dtype=torch.float32, device=dev)
        if use_fp8:
            rq = torch.empty((rows, H), dtype=torch.float8_e4m3fn, device=dev)
            rs = torch.empty((rows, H // 128), dtype=torch.float32, device=dev)
            quant = EP_QUANT_FP8_E4M3_1X128_POW2 if pow2_scales else EP_QUANT_FP8_E4M3_1X128
        else:
            rq = torch.empty((rows, H), dtype=torch.bfloat16, device=dev)
            rs = None
            quant = EP_QUANT_NONE
        _lib.ep_dispatch_dedup(x, topk_idx, topk_weights, self.num_experts, P, quant, rq, rs, ri,
                               rw, handle, self.workspace)
        event = self._event()
        if exact:
            R = int(handle.num_recv.item())
            rq, ri, rw = rq[:R], ri[:R], rw[:R]
            if rs is not None:
                rs = rs[:R]
        return ((rq, rs) if use_fp8 else rq), ri, rw, handle, event

    def combine_dedup(self, partition_out: torch.Tensor, handle: Layout):
        """Returns ``(y, event)``: y[t] = sum over the token's partitions of their rows."""
        T = handle.row_of.shape[0]
        H = partition_out.shape[-1]
        y = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)
        _lib.ep_combine_dedup(partition_out, handle, y, self.workspace)
        return y, self._event()

    # -------------------------------------------------- redundant experts --
    def lb_prefetch_weights(self, primary_of: torch.Tensor, weights: torch.Tensor):
        """Copy each primary slot's weights into its replica slots (in place);
        returns ``event``.  ``primary_of[s]`` names slot s's primary."""
        _lib.ep_lb_prefetch_weights(primary_of, weights, self.workspace)
        return self._event()

    def lb_reduce_grads(self, primary_of: torch.Tensor, grads: torch.Tensor):
        """Sum each primary's and its replicas' fp32 gradients (ascending slot
        order) into every member of the group (in place); returns ``event``."""
        _lib.ep_lb_reduce_grads(primary_of, grads, self.workspace)
        return self._event()

    # ----------------------------------------------------------- backward --
    def dispatch_backward(self, grad_recv_x: torch.Tensor, handle: Layout,
                          grad_recv_topk_weights: Optional[torch.Tensor] = None):
        """Returns ``(grad_x, grad_topk_weights or None, event)``."""
        T, K = handle.row_of.shape
        H = grad_recv_x.shape[-1]
        gx = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)
        gw = None
        if grad_recv_topk_weights is not None:
            gw = torch.empty((T, K), dtype=torch.float32, device=self.device)
        _lib.ep_dispatch_backward(grad_recv_x, handle, gx, self.workspace, grad_recv_topk_weights,
                                  gw)
        return gx, gw, self._event()

    def combine_backward(self, grad_y: torch.Tensor, expert_out: torch.Tensor, handle: Layout,
                         topk_weights: torch.Tensor):
        """Returns ``(grad_expert_out, grad_topk_weights, event)``; rows no slot names
        are left as zeros."""
        T, K = handle.row_of.shape
        geo = torch.zeros_like(expert_out)
        gw = torch.empty((T, K), dtype=torch.float32, device=self.device)
        _lib.ep_combine_backward(grad_y, expert_out, handle, topk_weights, geo, gw,
                                 self.workspace)
        return geo, gw, self._event()
