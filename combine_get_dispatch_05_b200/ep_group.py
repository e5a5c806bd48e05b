"""Expert parallelism across processes: partitions are ranks.

The DeepEP pages describe dispatch and combine as an exchange between the ranks of
an EP group ("DeepSeek 开源周第二弹：DeepEP", section "DeepEP 的常规内核和低延迟内核":
normal kernels over NVLink and RDMA; "deepseek-ai/DeepEP", section "典型工作流程":
dispatch, expert GEMM, combine back to the source ranks).  ``EpGroup`` offers two
transports, one process per GPU; rank r owns experts [r * E / W, (r + 1) * E / W).

``transport="peer"`` (GPUs of one node, NVLink / NVSwitch): every rank allocates one
IPC-shareable region (receive payload, scales, local ids, weights, expert outputs)
and maps every other rank's.  Per step:

  1. layout of this rank's tokens with P = W (one kernel);
  2. all-gather of every rank's per-expert counts (W x E int32);
  3. plan: where this rank's rows go in the owners' buffers (one kernel);
  4. dispatch: the FP8 (or BF16) rows, scales, local ids and weights are stored by
     the dispatch kernel straight into the owners' receive buffers over NVLink;
  5. a barrier (one-element all-reduce on the stream); the caller computes its
     experts into ``expert_out_buffer`` ...
  6. ... and combine: a barrier, then the combine kernel reads each token's expert
     outputs straight from the owners' buffers and reduces them in fixed k order.

  A rank receives its rows expert-major, then by source rank, then by source token
  and k: partition r's rows of the one-GPU dispatch of all ranks' tokens
  concatenated in rank order.

  ``dispatch(..., dedup=True)`` sends each token once to each rank that holds any of
  its experts (DeepEP's normal-kernel semantics; under group-limited routing about
  half the rows of the per-expert form cross NVLink): rows by source rank, then
  token, each with [K] local-id / weight lists (-1 / 0 for experts elsewhere); the
  caller writes one BF16 row per received row (its experts' weighted sum) into
  ``expert_out_buffer`` and combine sums the ranks' rows per token.

  ``low_latency_dispatch`` / ``low_latency_combine`` (constructed with
  ``ll_max_tokens``) use DeepEP's low-latency layout: per local expert, W blocks of
  ``ll_max_tokens`` rows, one per source rank, so the source writes each row and its
  counts straight to the owner with no exchange before the dispatch.

  ``return_recv_hook=True`` returns from a peer dispatch as soon as the rows are on
  their way, with a hook appended: the receive barrier, called when the rows are
  needed (work enqueued in between overlaps the transfer).

``transport="nccl"`` (any backend): the one-GPU dispatch with P = W fills a send
buffer whose rank-p rows are one contiguous slice; the rows, scales, local ids and
weights go to their owners with ``all_to_all_single`` (through host memory when the
backend is not NCCL), and the expert outputs come back the same way before the
one-GPU combine.  A rank receives its rows grouped by source rank, then expert.

Both return ``recv_counts_per_expert`` [W, E/W]: rows received from each source
rank for each local expert.
"""
from __future__ import annotations

from typing import List, Optional

import torch
import torch.distributed as dist

from . import _lib
from ._lib import EP_QUANT_FP8_E4M3_1X128, EP_QUANT_NONE, Layout

__all__ = ["EpGroup", "EpContext"]

_ALIGN = 256


class EpContext:
    """What combine needs from the dispatch that preceded it.

    The row counts are lists (and ``recv_rows`` an int) after a dispatch that
    synchronised with the host; after a peer dispatch with ``sync_sizes=False`` they
    stay on the device and the first read of ``send_counts``, ``recv_counts`` or
    ``recv_rows`` copies them to the host (one device synchronisation)."""

    def __init__(self, handle: Layout, send_counts, recv_counts, num_tokens: int, hidden: int,
                 topk_idx: Optional[torch.Tensor] = None,
                 dst_offset: Optional[torch.Tensor] = None, recv_rows=0,
                 order: str = "source_major", dedup: bool = False):
        self.handle = handle            # the sender-side layout (P = group size)
        self._send = send_counts        # rows this rank sent to each rank
        self._recv = recv_counts        # rows this rank received from each rank
        self.num_tokens = num_tokens
        self.hidden = hidden
        self.topk_idx = topk_idx        # peer transport only
        self.dst_offset = dst_offset
        self._recv_rows = recv_rows
        self.order = order
        self.dedup = dedup
        # True when the received tensors were cut to the received rows
        self.sizes_synced = isinstance(recv_rows, int)

    @staticmethod
    def _host(v):
        if callable(v):  # computed on first use (no-sync dispatch)
            v = v()
        return v.to("cpu").tolist() if isinstance(v, torch.Tensor) else v

    @property
    def send_counts(self) -> List[int]:
        self._send = self._host(self._send)
        return self._send

    @property
    def recv_counts(self) -> List[int]:
        self._recv = self._host(self._recv)
        return self._recv

    @property
    def recv_rows(self) -> int:
        if not isinstance(self._recv_rows, int):
            self._recv_rows = int(self.recv_rows_device.item())
        return self._recv_rows

    @property
    def recv_rows_device(self) -> Optional[torch.Tensor]:
        """The received row count as a device scalar (a no-sync peer dispatch; computed
        on the stream at the first read), else None."""
        if callable(self._recv_rows):
            self._recv_rows = self._recv_rows()
        return self._recv_rows if isinstance(self._recv_rows, torch.Tensor) else None


class EpGroup:
    """Dispatch / combine across the ranks of ``group`` (default: the world).

    transport: "nccl" (all-to-all collectives) or "peer" (the dispatch and combine
    kernels store to and load from the other GPUs' buffers; needs ``hidden``).
    capacity: rows of each rank's receive buffers in peer mode (default
    max_tokens * W * 8, every token of every rank routed here with top-8).
    num_topk: the largest K the peer buffers' id / weight lists hold (dedup rows).
    ll_max_tokens: peer transport, low-latency calls: the most tokens a rank sends
    per call (each rank's buffer holds E/W experts x W ranks x ll_max_tokens rows).
    Call :meth:`close` before destroying the process group.
    """

    def __init__(self, num_experts: int, group=None, max_tokens: int = 4096,
                 device: Optional[torch.device] = None, *, transport: str = "nccl",
                 hidden: Optional[int] = None, capacity: Optional[int] = None,
                 num_topk: int = 8, ll_max_tokens: int = 0):
        self.group = group if group is not None else dist.group.WORLD
        self.world = dist.get_world_size(self.group)
        self.rank = dist.get_rank(self.group)
        if num_experts % self.world:
            raise ValueError("num_experts must be a multiple of the group size")
        if transport not in ("nccl", "peer"):
            raise ValueError(f"unknown transport {transport!r}")
        self.transport = transport
        self.num_experts = num_experts
        self.experts_per_rank = num_experts // self.world
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.max_tokens = max_tokens
        self.workspace = self._new_workspace(max_tokens)
        self.via_host = dist.get_backend(self.group) != "nccl"
        self._peer = None
        if transport == "peer":
            if hidden is None:
                raise ValueError("the peer transport needs `hidden` to size the receive buffers")
            self._open_peers(int(hidden), int(capacity if capacity is not None
                                                  else max_tokens * self.world * 8),
                             int(num_topk), int(ll_max_tokens))

    def _new_workspace(self, tokens: int) -> torch.Tensor:
        ws = torch.empty(_lib.ep_workspace_bytes(max(tokens, 1), self.num_experts, self.world),
                         dtype=torch.uint8, device=self.device)
        _lib.ep_workspace_init(ws)
        return ws

    # ---------------------------------------------------------- peer buffers --
    def _map_region(self, sizes) -> dict:
        """Allocate this rank's IPC region holding the named arrays (each 256-byte
        aligned), exchange the handles and map every other rank's region.  Returns
        the region's description with every rank's array addresses."""
        offsets, total = {}, 0
        for name, n in sizes:
            offsets[name] = total
            total += (n + _ALIGN - 1) // _ALIGN * _ALIGN
        total = max(total, _ALIGN)
        base, handle = _lib.ep_ipc_alloc(total)
        handles: List[bytes] = [b""] * self.world
        dist.all_gather_object(handles, handle, group=self.group)
        bases, opened = [], []
        try:
            for q, h in enumerate(handles):
                if q == self.rank:
                    bases.append(base)
                else:
                    ptr = _lib.ep_ipc_open(h)
                    opened.append(ptr)
                    bases.append(ptr)
        except Exception:
            for ptr in opened:
                _lib.ep_ipc_close(ptr)
            _lib.ep_ipc_free(base)
            raise
        self._regions.append(dict(base=base, opened=opened))
        return dict(region=_lib.device_bytes(base, total, self.device), offsets=offsets,
                    sizes=dict(sizes),
                    addrs={n: [b + offsets[n] for b in bases] for n, _ in sizes})

    def _open_peers(self, hidden: int, capacity: int, topk: int, ll_max_tokens: int) -> None:
        """The normal region: recv_x (room for BF16 rows) | recv_scales | recv_topk_idx |
        recv_topk_weights (room for [K] lists) | expert_out; and, with ll_max_tokens,
        the low-latency region: [E/W, W*cap] rows of E4M3 payload, scales and BF16
        outputs, and the [E/W, W] counts."""
        if hidden % 128:
            raise ValueError("hidden must be a multiple of 128")
        self._regions = []
        self._views = {}
        self._flag = torch.zeros(1, dtype=torch.int32, device=self.device)
        sizes = [("recv_x", capacity * hidden * 2), ("recv_scales", capacity * (hidden // 128) * 4),
                 ("recv_topk_idx", capacity * topk * 4), ("recv_topk_weights", capacity * topk * 4),
                 ("expert_out", capacity * hidden * 2)]
        reg = self._map_region(sizes)
        self._peer = dict(reg, hidden=hidden, capacity=capacity, topk=topk, ll=None)
        self.tables = _lib.PeerTables.from_addresses(
            self.device, capacity, *[reg["addrs"][n] for n, _ in sizes])
        if ll_max_tokens > 0:
            rows = self.experts_per_rank * self.world * ll_max_tokens
            ll = self._map_region([("x", rows * hidden), ("scales", rows * (hidden // 128) * 4),
                                   ("count", self.experts_per_rank * self.world * 4),
                                   ("expert_out", rows * hidden * 2)])
            ll["cap"] = ll_max_tokens
            ll["tables"] = {n: torch.tensor(a, dtype=torch.int64, device=self.device)
                            for n, a in ll["addrs"].items()}
            self._peer["ll"] = ll

    def _view(self, name: str, dtype, shape, region=None) -> torch.Tensor:
        """A typed view of a named array of a region; made once per (array, dtype,
        shape) and kept, as every call of a step asks for the same views.  Each call
        returns a fresh alias of the kept view, so that in-place changes of a
        returned tensor's shape do not reach later calls."""
        pr = self._peer if region is None else region
        key = (id(pr), name, dtype, tuple(shape))
        v = self._views.get(key)
        if v is None:
            n = 1
            for d in shape:
                n *= d
            n *= torch.empty(0, dtype=dtype).element_size()
            o = pr["offsets"][name]
            v = self._views[key] = pr["region"][o:o + n].view(dtype).view(*shape)
        return v.detach()

    def _stream(self):
        """The current stream of this group's device, resolved once per call and
        passed to every library call of it."""
        if self.device.type != "cuda":
            return None
        if _lib._raw_stream is not None:
            return _lib._raw_stream(self.device.index)
        return torch.cuda.current_stream(self.device).cuda_stream

    @staticmethod
    def _rows(t: torch.Tensor, n: int) -> torch.Tensor:
        return t if n == t.shape[0] else t[:n]

    def expert_out_buffer(self, ctx: EpContext) -> torch.Tensor:
        """Peer transport: the BF16 [recv rows, H] buffer the expert outputs go into
        (row i answers received row i); the other ranks' combine kernels read it.
        After a dispatch with sync_sizes=False: all [capacity, H] rows (the first
        ctx.recv_rows_device of them are read)."""
        if self._peer is None:
            raise RuntimeError("expert_out_buffer belongs to the peer transport")
        cap, H = self._peer["capacity"], self._peer["hidden"]
        full = self._view("expert_out", torch.bfloat16, (cap, H))
        return full[:ctx.recv_rows] if ctx.sizes_synced else full

    def close(self) -> None:
        """Unmap the peers' regions and free this rank's (a collective: every rank
        calls it, after its last combine)."""
        if self._peer is None:
            return
        self._host_barrier()  # no rank's kernels touch any region any more
        for reg in self._regions:
            for ptr in reg["opened"]:
                _lib.ep_ipc_close(ptr)
        self._host_barrier()  # every rank has closed its mappings of this rank's regions
        self._peer = None
        self._views = {}
        for reg in self._regions:
            _lib.ep_ipc_free(reg["base"])
        self._regions = []

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

    def _all_gather_rows(self, t: torch.Tensor) -> torch.Tensor:
        """[n] on every rank -> [W, n] in rank order."""
        if not self.via_host:
            out = torch.empty((self.world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
            dist.all_gather_into_tensor(out, t.contiguous(), group=self.group)
            return out
        parts = [torch.empty_like(t, device="cpu") for _ in range(self.world)]
        dist.all_gather(parts, t.contiguous().cpu(), group=self.group)
        return torch.stack(parts).to(t.device)

    def _barrier(self) -> None:
        """Every rank's preceding work on the stream is done before anything after it
        on the stream (NCCL: asynchronous for the host)."""
        if not self.via_host:
            dist.all_reduce(self._flag, group=self.group)  # ordered on the current stream
        else:
            if self.device.type == "cuda":
                torch.cuda.synchronize(self.device)
            dist.barrier(group=self.group)

    def _host_barrier(self) -> None:
        """As _barrier, and the host waits for it: when it returns, every rank's host
        has reached this point and every rank's preceding device work is done."""
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)
        self._barrier()
        if self.device.type == "cuda":
            torch.cuda.synchronize(self.device)

    # --------------------------------------------------------------- dispatch --
    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                 use_fp8: bool = True, dedup: bool = False, return_recv_hook: bool = False,
                 sync_sizes: bool = True):
        """Returns ``(recv_x, recv_local_idx, recv_weights, recv_counts_per_expert, ctx)``.

        recv_x: ``(float8_e4m3fn [Rr, H], float32 [Rr, H/128])`` or BF16 ``[Rr, H]``;
        recv_local_idx: int32 [Rr] (expert id minus this rank's first expert);
        recv_weights: float32 [Rr]; recv_counts_per_expert: int32 [W, E/W] rows
        received from each source rank for each local expert.  Row order: see the
        module docstring (``ctx.order``).

        dedup (peer transport): one row per (token, rank); recv_local_idx and
        recv_weights are [Rr, K] lists and the counts are [W, 1] rows per source.

        sync_sizes=False (peer transport): nothing waits on the host.  The counts stay
        on the device (the all-gather, the plan and the dispatch are all enqueued on
        the stream), the received tensors are [capacity, ...] views of which the first
        ``ctx.recv_rows_device`` rows are this step's, and a receiver over capacity is
        not raised on the host: its rows are dropped by the dispatch kernel and
        reported as EP_DEV_CAPACITY in the workspace status.  (DeepEP likewise returns
        exact-size tensors only after a host wait.)

        return_recv_hook (peer transport): return as soon as this rank's rows are on
        their way, with a ``hook`` appended to the result; calling it (every rank, a
        collective) waits until every rank's rows have landed.  Work enqueued
        between the two overlaps the transfer; the received tensors are valid after
        the hook.  As DeepEP's receive hook ("deepseek.csdn.net/67bd3eb22e30c863900615cc",
        "推理解码阶段的应用": low_latency_dispatch returns a hook).
        """
        if return_recv_hook and self.transport != "peer":
            raise NotImplementedError("the receive hook belongs to the peer transport")
        if not sync_sizes and self.transport != "peer":
            raise NotImplementedError("the all-to-all needs its splits on the host")
        T = x.shape[0]
        if T > self.max_tokens:
            self.max_tokens = T
            self.workspace = self._new_workspace(T)
        if dedup:
            if self.transport != "peer":
                raise NotImplementedError("deduplicated rows are offered by the peer transport")
            return self._deliver(
                self._dispatch_peer_dedup(x, topk_idx, topk_weights, use_fp8, sync_sizes),
                return_recv_hook)
        if self.transport == "peer":
            return self._deliver(self._dispatch_peer(x, topk_idx, topk_weights, use_fp8, sync_sizes),
                                 return_recv_hook)
        return self._dispatch_nccl(x, topk_idx, topk_weights, use_fp8)

    def _dispatch_nccl(self, x, topk_idx, topk_weights, use_fp8):
        T, H = x.shape
        K = topk_idx.shape[1]
        W, E, epp = self.world, self.num_experts, self.experts_per_rank
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
        ctx = EpContext(lay, send_counts, recv_counts, T, H, recv_rows=Rr)
        recv_x = (recv_q.view(torch.float8_e4m3fn), recv_s) if use_fp8 else recv_q
        return recv_x, recv_i, recv_w, per_expert, ctx

    def _dispatch_peer(self, x, topk_idx, topk_weights, use_fp8, sync_sizes=True):
        T, H = x.shape
        K = topk_idx.shape[1]
        W, E, epp, r = self.world, self.num_experts, self.experts_per_rank, self.rank
        pr = self._peer
        if H != pr["hidden"]:
            raise ValueError(f"hidden {H} differs from the receive buffers' {pr['hidden']}")
        cap, dev, st = pr["capacity"], self.device, self._stream()
        lay = Layout.empty(T, K, E, W, dev)
        _lib.ep_get_dispatch_layout(topk_idx, E, W, lay, self.workspace, stream=st)
        counts = self._all_gather_rows(lay.num_tokens_per_expert)  # [W, E]
        if sync_sizes:
            # every rank reads the same counts: all of them raise, or none
            totals = counts.view(W, W, epp).sum(dim=(0, 2)).to("cpu").tolist()
            if max(totals) > cap:
                raise ValueError(f"a rank would receive {max(totals)} rows; capacity is {cap}")
        dst = torch.empty(E, dtype=torch.int32, device=dev)
        rc = torch.empty(epp, dtype=torch.int32, device=dev)
        ro = torch.empty(epp + 1, dtype=torch.int32, device=dev)
        _lib.ep_peer_plan(counts, r, lay.expert_offset, cap, dst, rc, ro, self.workspace,
                          stream=st)
        quant = EP_QUANT_FP8_E4M3_1X128 if use_fp8 else EP_QUANT_NONE
        _lib.ep_peer_dispatch(x, topk_idx, topk_weights, E, W, quant, lay, dst, self.tables,
                              self.workspace, stream=st)
        per_expert = counts[:, r * epp:(r + 1) * epp]
        if sync_sizes:
            Rr = int(totals[r])
            send = counts.view(W, W, epp)[r].sum(dim=1).to("cpu").tolist()
            recv = per_expert.sum(dim=1).to("cpu").tolist()
        else:  # reductions launched only if the caller reads them
            Rr = lambda: per_expert.sum()  # noqa: E731
            send = lambda: counts.view(W, W, epp)[r].sum(dim=1)  # noqa: E731
            recv = lambda: per_expert.sum(dim=1)  # noqa: E731
        n = Rr if sync_sizes else cap
        ctx = EpContext(lay, send, recv, T, H, topk_idx=topk_idx, dst_offset=dst, recv_rows=Rr,
                        order="expert_major")
        ri = self._rows(self._view("recv_topk_idx", torch.int32, (cap,)), n)
        rw = self._rows(self._view("recv_topk_weights", torch.float32, (cap,)), n)
        if use_fp8:
            recv_x = (self._rows(self._view("recv_x", torch.float8_e4m3fn, (cap, H)), n),
                      self._rows(self._view("recv_scales", torch.float32, (cap, H // 128)), n))
        else:
            recv_x = self._rows(self._view("recv_x", torch.bfloat16, (cap, H)), n)
        return recv_x, ri, rw, per_expert, ctx

    def _dispatch_peer_dedup(self, x, topk_idx, topk_weights, use_fp8, sync_sizes=True):
        T, H = x.shape
        K = topk_idx.shape[1]
        W, E, r = self.world, self.num_experts, self.rank
        pr = self._peer
        if H != pr["hidden"]:
            raise ValueError(f"hidden {H} differs from the receive buffers' {pr['hidden']}")
        if K > pr["topk"]:
            raise ValueError(f"top-k {K} exceeds the buffers' lists of {pr['topk']}")
        if W > 32:
            raise ValueError("deduplicated rows support at most 32 ranks")
        cap, dev, st = pr["capacity"], self.device, self._stream()
        lay = Layout.empty(T, W, W, W, dev)  # partition-sized handle
        _lib.ep_get_dispatch_layout_dedup(topk_idx, E, W, lay, self.workspace, stream=st)
        counts = self._all_gather_rows(lay.num_tokens_per_expert)  # [W sources, W owners]
        if sync_sizes:
            totals = counts.sum(dim=0).to("cpu").tolist()
            if max(totals) > cap:
                raise ValueError(f"a rank would receive {max(totals)} rows; capacity is {cap}")
        dst = torch.empty(W, dtype=torch.int32, device=dev)
        rc = torch.empty(1, dtype=torch.int32, device=dev)
        ro = torch.empty(2, dtype=torch.int32, device=dev)
        _lib.ep_peer_plan(counts, r, lay.expert_offset, cap, dst, rc, ro, self.workspace,
                          stream=st)
        quant = EP_QUANT_FP8_E4M3_1X128 if use_fp8 else EP_QUANT_NONE
        _lib.ep_peer_dispatch_dedup(x, topk_idx, topk_weights, E, W, quant, lay, dst, self.tables,
                                    self.workspace, stream=st)
        per_source = counts[:, r:r + 1]
        send, recv = counts[r], per_source.reshape(-1)
        if sync_sizes:
            Rr = int(totals[r])
            send, recv = send.to("cpu").tolist(), recv.to("cpu").tolist()
        else:  # the reduction is launched only if the caller reads it
            Rr = lambda: per_source.sum()  # noqa: E731
        n = Rr if sync_sizes else cap
        ctx = EpContext(lay, send, recv, T, H, dst_offset=dst, recv_rows=Rr, order="source_major",
                        dedup=True)
        ri = self._rows(self._view("recv_topk_idx", torch.int32, (cap, K)), n)
        rw = self._rows(self._view("recv_topk_weights", torch.float32, (cap, K)), n)
        if use_fp8:
            recv_x = (self._rows(self._view("recv_x", torch.float8_e4m3fn, (cap, H)), n),
                      self._rows(self._view("recv_scales", torch.float32, (cap, H // 128)), n))
        else:
            recv_x = self._rows(self._view("recv_x", torch.bfloat16, (cap, H)), n)
        return recv_x, ri, rw, per_source, ctx

    # ------------------------------------------------------------ low latency --
    def _deliver(self, result, return_recv_hook: bool):
        """The receive side of a peer dispatch: a barrier after which every rank's
        rows have landed in their owners' buffers, now or when the hook is called."""
        if not return_recv_hook:
            self._barrier()
            return result
        done = []

        def hook() -> None:
            if not done:  # once
                done.append(True)
                self._barrier()

        return result + (hook,)

    def low_latency_dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor,
                             return_recv_hook: bool = False):
        """Peer transport (constructed with ll_max_tokens): DeepEP's low-latency
        dispatch across the ranks.  Every rank's FP8 rows go straight into padded
        per-expert blocks of their owners' buffers, with no count exchange first.

        Returns ``((recv_x, recv_scales), recv_count, ctx)``: recv_x E4M3
        [E/W, W*cap, H] and recv_scales [E/W, W*cap, H/128] (rows [s*cap, s*cap + n)
        of local expert el come from rank s, n = recv_count[el, s]), recv_count int32
        [E/W, W]; with return_recv_hook, a ``hook`` as for :meth:`dispatch`."""
        ll = self._peer["ll"] if self._peer is not None else None
        if ll is None:
            raise RuntimeError("low-latency calls need the peer transport and ll_max_tokens")
        T, H = x.shape
        K = topk_idx.shape[1]
        cap, E, W, epp = ll["cap"], self.num_experts, self.world, self.experts_per_rank
        if T > cap:
            raise ValueError(f"{T} tokens exceed ll_max_tokens = {cap}")
        h = _lib.LowLatencyHandle.empty(T, K, E, cap, self.device)
        t = ll["tables"]
        _lib.ep_peer_low_latency_dispatch(x, topk_idx, cap, E, W, self.rank, t["x"], t["scales"],
                                          t["count"], h, self.workspace, stream=self._stream())
        rows = epp * W * cap
        q = self._view("x", torch.float8_e4m3fn, (epp, W * cap, H), ll)
        s = self._view("scales", torch.float32, (epp, W * cap, H // 128), ll)
        count = self._view("count", torch.int32, (epp, W), ll)
        ctx = EpContext(h, [], [], T, H, topk_idx=topk_idx, recv_rows=rows, order="low_latency")
        return self._deliver(((q, s), count, ctx), return_recv_hook)

    def ll_expert_out_buffer(self) -> torch.Tensor:
        """BF16 [E/W, W*cap, H]: where a rank's low-latency expert outputs go (row i of
        a block answers received row i); the other ranks' combines read it."""
        ll = self._peer["ll"]
        return self._view("expert_out", torch.bfloat16,
                          (self.experts_per_rank, self.world * ll["cap"], self._peer["hidden"]), ll)

    def low_latency_combine(self, expert_out: torch.Tensor, ctx: EpContext,
                            topk_weights: torch.Tensor) -> torch.Tensor:
        """expert_out: the tensor from :meth:`ll_expert_out_buffer`.  Returns y BF16
        [T, H]: each token's expert outputs, read from their owners and reduced in
        fixed k order with its weights."""
        if expert_out.data_ptr() != self.ll_expert_out_buffer().data_ptr():
            raise ValueError("write the expert outputs into ll_expert_out_buffer()")
        y = torch.empty((ctx.num_tokens, ctx.hidden), dtype=torch.bfloat16, device=self.device)
        self._barrier()  # every rank's expert outputs are complete
        _lib.ep_peer_low_latency_combine(self._peer["ll"]["tables"]["expert_out"], ctx.topk_idx,
                                         ctx.handle, topk_weights, y, self.num_experts, self.world,
                                         self.rank, self.workspace, stream=self._stream())
        return y

    # ---------------------------------------------------------------- combine --
    def combine(self, expert_out: torch.Tensor, ctx: EpContext,
                topk_weights: torch.Tensor) -> torch.Tensor:
        """expert_out: BF16 [recv rows, H] in the received row order (peer transport:
        the tensor from :meth:`expert_out_buffer`).  Returns y: BF16 [T, H], the
        weighted sum of each token's expert outputs."""
        y = torch.empty((ctx.num_tokens, ctx.hidden), dtype=torch.bfloat16, device=self.device)
        if self.transport == "peer":
            # checked on every rank alike (also with no rows), before the barrier
            if expert_out.data_ptr() != self.expert_out_buffer(ctx).data_ptr():
                raise ValueError("write the expert outputs into expert_out_buffer(ctx)")
            self._barrier()  # every rank's expert outputs are complete
            st = self._stream()
            if ctx.dedup:  # partition outputs are already weighted: a plain sum
                _lib.ep_peer_combine_dedup(self.tables, ctx.handle, ctx.dst_offset, y, self.world,
                                           self.workspace, stream=st)
            else:
                _lib.ep_peer_combine(self.tables, ctx.handle, ctx.topk_idx, ctx.dst_offset,
                                     topk_weights, y, self.num_experts, self.world,
                                     self.workspace, stream=st)
            return y
        Rs = sum(ctx.send_counts)
        back = self._a2a(expert_out, Rs, ctx.send_counts, ctx.recv_counts)
        if Rs == 0:
            back = torch.zeros((1, ctx.hidden), dtype=torch.bfloat16, device=self.device)
        _lib.ep_combine(back, ctx.handle, topk_weights, y, self.workspace)
        return y
