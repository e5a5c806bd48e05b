"""Expert parallelism across processes: partitions are ranks.

The DeepEP pages describe dispatch and combine as an all-to-all between the
ranks of an EP group ("DeepSeek 开源周第二弹：DeepEP", section "DeepEP 的常规内核和低延迟
内核": normal kernels over NVLink and RDMA; "deepseek-ai/DeepEP", section "典型工作流程":
dispatch, expert GEMM, combine back to the source ranks).  ``EpGroup`` builds that
exchange from this library's one-GPU kernels and ``torch.distributed``:

dispatch (on every rank, for its own tokens)
  1. layout + FP8 (or BF16) dispatch with P = group size: the rows for rank p are
     one contiguous, expert-major slice of the send buffer (partition p);
  2. the per-rank row counts (from the layout's expert offsets) are exchanged;
  3. rows, scales, local expert ids and weights go to their owner ranks with
     ``all_to_all_single`` (NCCL on GPUs; other backends through host memory).
  Each rank receives, per source rank in rank order, that source's rows for its
  own experts (expert-major within a source), plus per-(source, local expert)
  counts for the expert computation.
combine
  4. the expert outputs go back along the same splits, so each row lands where
     it left the sender's send buffer;
  5. the one-GPU combine kernel reduces them with the sender's handle.

The exchange is the plain collective; the kernels are the library's.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch
import torch.distributed as dist

from . import _lib
from ._lib import EP_QUANT_FP8_E4M3_1X128, EP_QUANT_NONE, Layout

__all__ = ["EpGroup", "EpContext"]


@dataclass
class EpContext:
    """What combine needs from the dispatch that preceded it."""

    handle: Layout               # the sender-side layout (P = group size)
    send_counts: List[int]       # rows this rank sent to each rank
    recv_counts: List[int]       # rows this rank received from each rank
    num_tokens: int
    hidden: int


class EpGroup:
    """Dispatch / combine across the ranks of ``group`` (default: the world).

    Rank r owns experts [r * E / W, (r + 1) * E / W).  One process per GPU.
    """

    def __init__(self, num_experts: int, group=None, max_tokens: int = 4096,
                 device: Optional[torch.device] = None):
        self.group = group if group is not None else dist.group.WORLD
        self.world = dist.get_world_size(self.group)
        self.rank = dist.get_rank(self.group)
        if num_experts % self.world:
            raise ValueError("num_experts must be a multiple of the group size")
        self.num_experts = num_experts
        self.experts_per_rank = num_experts // self.world
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.max_tokens = max_tokens
        self.workspace = self._new_workspace(max_tokens)
        self.via_host = dist.get_backend(self.group) != "nccl"

    def _new_workspace(self, tokens: int) -> torch.Tensor:
        ws = torch.empty(_lib.ep_workspace_bytes(max(tokens, 1), self.num_experts, self.world),
                         dtype=torch.uint8, device=self.device)
        _lib.ep_workspace_init(ws)
        return ws

    # --------------------------------------------------------------- exchange --
    def _a2a(self, inp: torch.Tensor, out_rows: int, out_splits: List[int],
             in_splits: List[int]) -> torch.Tensor:
        """all_to_all_single along dim 0 (rows); through host memory unless NCCL."""
        shape = (out_rows,) + tuple(inp.shape[1:])
        if not self.via_host:
            out = torch.empty(shape, dtype=inp.dtype, device=inp.device)
            dist.all_to_all_single(out, inp.contiguous(), out_splits, in_splits, group=self.group)
            return out
        out = torch.empty(shape, dtype=inp.dtype)
        dist.all_to_all_single(out, inp.contiguous().cpu(), out_splits, in_splits,
                               group=self.group)
        return out.to(inp.device)

    # --------------------------------------------------------------- dispatch --
    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                 use_fp8: bool = True):
        """Returns ``(recv_x, recv_local_idx, recv_weights, recv_counts_per_expert, ctx)``.

        recv_x: ``(float8_e4m3fn [Rr, H], float32 [Rr, H/128])`` or BF16 ``[Rr, H]``;
        recv_local_idx: int32 [Rr] (expert id minus this rank's first expert);
        recv_weights: float32 [Rr]; recv_counts_per_expert: int32 [W, E/W] rows
        received from each source rank for each local expert (rows are grouped by
        source rank, then local expert, then source token).
        """
        T, H = x.shape
        K = topk_idx.shape[1]
        W, E, epp = self.world, self.num_experts, self.experts_per_rank
        if T > self.max_tokens:
            self.max_tokens = T
            self.workspace = self._new_workspace(T)
        rows = max(T * K, 1)
        dev = self.device
        lay = Layout.empty(T, K, E, W, dev)
        ri = torch.empty(rows, dtype=torch.int32, device=dev)
        rw = torch.empty(rows, dtype=torch.float32, device=dev)
        if use_fp8:
            q = torch.empty((rows, H), dtype=torch.uint8, device=dev)
            s = torch.empty((rows, H // 128), dtype=torch.float32, device=dev)
            _lib.ep_dispatch(x, topk_idx, topk_weights, E, W, EP_QUANT_FP8_E4M3_1X128, q, s, ri,
                             rw, lay, self.workspace)
        else:
            q = torch.empty((rows, H), dtype=torch.bfloat16, device=dev)
            s = None
            _lib.ep_dispatch(x, topk_idx, topk_weights, E, W, EP_QUANT_NONE, q, None, ri, rw,
                             lay, self.workspace)
        # rows per destination rank: partition p = rows [offset[p*epp], offset[(p+1)*epp])
        bounds = lay.expert_offset[::epp].to("cpu").tolist()  # W + 1 values (synchronises)
        send_counts = [bounds[p + 1] - bounds[p] for p in range(W)]
        counts_dev = torch.tensor(send_counts, dtype=torch.int64, device=dev)
        recv_counts = self._a2a(counts_dev, W, [1] * W, [1] * W).to("cpu").tolist()
        Rs, Rr = sum(send_counts), sum(recv_counts)
        recv_q = self._a2a(q[:Rs], Rr, recv_counts, send_counts)
        recv_s = self._a2a(s[:Rs], Rr, recv_counts, send_counts) if use_fp8 else None
        recv_i = self._a2a(ri[:Rs], Rr, recv_counts, send_counts)
        recv_w = self._a2a(rw[:Rs], Rr, recv_counts, send_counts)
        per_expert = self._a2a(lay.num_tokens_per_expert.view(W, epp), W, [1] * W, [1] * W)
        ctx = EpContext(lay, send_counts, recv_counts, T, H)
        recv_x = (recv_q.view(torch.float8_e4m3fn), recv_s) if use_fp8 else recv_q
        return recv_x, recv_i, recv_w, per_expert, ctx

    # ---------------------------------------------------------------- combine --
    def combine(self, expert_out: torch.Tensor, ctx: EpContext,
                topk_weights: torch.Tensor) -> torch.Tensor:
        """expert_out: BF16 [sum(recv_counts), H] in the received row order.
        Returns y: BF16 [T, H], the weighted sum of each token's expert outputs."""
        Rs = sum(ctx.send_counts)
        back = self._a2a(expert_out, Rs, ctx.send_counts, ctx.recv_counts)
        if Rs == 0:
            back = torch.zeros((1, ctx.hidden), dtype=torch.bfloat16, device=self.device)
        y = torch.empty((ctx.num_tokens, ctx.hidden), dtype=torch.bfloat16, device=self.device)
        _lib.ep_combine(back, ctx.handle, topk_weights, y, self.workspace)
        return y
