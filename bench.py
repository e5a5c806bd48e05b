#!/usr/bin/env python
"""Benchmark of the MoE dispatch / combine hot path on B200.

One step = one pass of the whole path over one batch of the "normal" workload
(4096 tokens x hidden 7168, top-8 of 256 experts in 8 logical partitions with
top-4-group routing): routing layout + FP8 dispatch (3 kernels, one call) and
BF16 combine (1 kernel, one call).  The expert computation between them is out
of scope; combine reads expert outputs prepared once before timing (the
dispatched rows dequantised, i.e. identity experts).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  `value` is algorithmic HBM GB/s of the whole
step (bytes the method must move / device time, summed over ranks' batches,
max time over ranks).  Steps are captured in CUDA graphs, ten whole steps (the
layout, dispatch and combine kernels of each) per graph by default
(`--steps-per-graph`), and timed with CUDA events on the launching stream around
each replay; a second pass times the dispatch and the combine apart (two graphs,
events between them) for the breakdown, and a third the whole step as one graph
per step.  Steps run back
to back: every step reads 529 MB of inputs (x and the expert outputs) and
writes 294 MB, several times the 126 MB L2, so nothing a step reads is still in
L2 from the step before.  `--l2-flush write|read` instead flushes L2 with a
256 MiB buffer before every step (outside the events).
`--impl reference` times the CPU oracle on the host's cores instead (the same
workload, or a bounded prefix of it when the host is slow).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dispatch/combine HBM GB/s (% of B200 peak) at 4096x7168 top-8; LL latency µs"
DTYPE_TEXT = {True: "f32 arithmetic; fp8-e4m3 dispatch payload, bf16 combine",
              False: "f32 arithmetic; bf16 dispatch payload, bf16 combine"}

WORKLOAD_TEXT = {
    "normal": "normal: 4096 tokens x hidden 7168 BF16, top-8 of 256 experts in 8 logical "
              "partitions, top-4-of-8-group routing, FP8 (E4M3, 1x128 scales) dispatch + BF16 "
              "combine",
    "skew": "skew: 4096 tokens x hidden 7168, top-8 of 256 experts (Zipf 1.2 popularity, 5% "
            "of slots masked), FP8 dispatch + BF16 combine",
    "bf16": "bf16: 8192 tokens x hidden 4096, top-6 of 64 experts in 16 partitions, 1% "
            "outlier rows, BF16 dispatch (no quantisation) + BF16 combine",
    "stress": "stress: 32768 tokens x hidden 7168, top-8 over 288 expert slots (256 + 32 "
              "replicas) in 8 partitions, FP8 dispatch + BF16 combine",
}
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ helpers --

def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(T, H, K, E, P, R, fp8: bool):
    """Bytes the method must move: reads of inputs and writes of outputs,
    once each; no padding, no unwritten worst-case rows."""
    payload = R * H * (1 if fp8 else 2)
    scales = R * (H // 128) * 4 if fp8 else 0
    meta = (T * K * 8 + T * K * 4          # topk_idx, topk_weights read
            + R * 4 + R * 4                # recv_topk_idx, recv_topk_weights
            + R * 4 + T * K * 4            # src_of, row_of
            + (E + 1) * 4 + E * 4 + P * 4  # offsets, counts
            + T * P)                       # is_token_in_partition
    dispatch = T * H * 2 + payload + scales + meta
    combine = R * H * 2 + T * H * 2 + T * K * 8
    return dispatch, combine


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the benchmark runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = vis.split(",")[local_rank] if vis else str(local_rank)
        self.idx = idx.strip()
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", self.idx], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        self.start_time = time.time()

    def mark(self, t0, t1):
        self.t0, self.t1 = t0, t1

    def stop(self):
        if self.proc is None:
            return None
        end = time.time()
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        if not rows:
            return None
        # samples are evenly spaced over [start_time, end]: keep those inside the timed window
        n = len(rows)
        ts = [self.start_time + (end - self.start_time) * (i + 0.5) / n for i in range(n)]
        sel = [r for r, t in zip(rows, ts) if self.t0 is not None and self.t0 <= t <= self.t1]
        window = "timed region"
        if not sel:
            sel, window = rows, "whole run (timed region shorter than the sampling period)"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        mhz, maxmhz = [], []
        for r in sel:
            try:
                mhz.append(float(r[1]))
                maxmhz.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxmhz),
                "reasons": sorted(reasons), "samples": len(mhz), "window": window}


def source_hash(paths):
    """Hash of the code in `paths` with comments and blank space removed, so that
    a comment edit does not invalidate a capture of the same kernel."""
    import re

    h = hashlib.sha256()
    for p in paths:
        text = open(os.path.join(ROOT, p), encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)  # block comments
        text = re.sub(r"//[^\n]*", " ", text)                # line comments
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


COMBINE_SOURCES = ["combine_get_dispatch_05_b200/csrc/combine.cu",
                   "combine_get_dispatch_05_b200/csrc/ep_device.cuh"]
DISPATCH_SOURCES = ["combine_get_dispatch_05_b200/csrc/dispatch.cu",
                    "combine_get_dispatch_05_b200/csrc/ep_quant.cuh",
                    "combine_get_dispatch_05_b200/csrc/ep_device.cuh",
                    "combine_get_dispatch_05_b200/csrc/ep_internal.h"]
LAYOUT_SOURCES = ["combine_get_dispatch_05_b200/csrc/layout.cu",
                  "combine_get_dispatch_05_b200/csrc/ep_device.cuh",
                  "combine_get_dispatch_05_b200/csrc/ep_internal.h"]


def profiled_traffic(summary: str, sources):
    """dram bytes per launch from a committed ncu summary, if it was taken on the
    current source of the kernel (else None)."""
    p = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(p):
        return None
    vals = {}
    for line in open(p):
        if ":" in line and line.startswith("- "):
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    try:
        if vals.get("source_sha256") != source_hash(sources):
            return None
        return int(float(vals["dram_bytes_per_full_launch"]))
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------- our path -----

class PathRunner:
    """Device buffers and CUDA graphs for one workload's dispatch + combine."""

    def __init__(self, ep, w, dev, use_graphs=True):
        import numpy as np
        import torch

        self.ep, self.w, self.dev = ep, w, dev
        T, H, K, E, P = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
        self.T, self.H, self.K, self.E, self.P = T, H, K, E, P
        self.fp8 = w.quant == "fp8"
        self.quant = ep.EP_QUANT_FP8_E4M3_1X128 if self.fp8 else ep.EP_QUANT_NONE
        self.x = torch.from_numpy(w.x.view(np.int16)).to(dev).view(torch.bfloat16)
        self.idx = torch.from_numpy(w.topk_idx).to(dev)
        self.wts = torch.from_numpy(w.topk_weights).to(dev)
        rows = max(T * K, 1)
        self.recv_q = torch.empty((rows, H), dtype=torch.uint8 if self.fp8 else torch.bfloat16,
                                  device=dev)
        self.recv_s = torch.empty((rows, H // 128), dtype=torch.float32, device=dev) \
            if self.fp8 else None
        self.recv_i = torch.empty(rows, dtype=torch.int32, device=dev)
        self.recv_w = torch.empty(rows, dtype=torch.float32, device=dev)
        self.lay = ep.Layout.empty(T, K, E, P, dev)
        self.ws = torch.empty(ep.ep_workspace_bytes(T, E, P), dtype=torch.uint8, device=dev)
        ep.ep_workspace_init(self.ws)
        self.y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.dispatch()
        torch.cuda.synchronize()
        self.R = int(self.lay.num_recv.item())
        if self.fp8:
            q = self.recv_q.view(torch.float8_e4m3fn).to(torch.float32)
            self.eo = (q * self.recv_s.repeat_interleave(128, dim=1)).to(torch.bfloat16)
            del q
        else:
            self.eo = self.recv_q.clone()
        self.combine()
        torch.cuda.synchronize()
        if ep.ep_read_status(self.ws) != 0:
            raise RuntimeError("device status set during setup")
        self.bytes_dispatch, self.bytes_combine = algorithmic_bytes(T, H, K, E, P, self.R, self.fp8)
        self.graphs = None
        self._step_graphs = {}
        if use_graphs:
            self.graphs = self._capture()

    def dispatch(self, stream=None):
        self.ep.ep_dispatch(self.x, self.idx, self.wts, self.E, self.P, self.quant, self.recv_q,
                            self.recv_s, self.recv_i, self.recv_w, self.lay, self.ws, stream)

    def combine(self, stream=None):
        self.ep.ep_combine(self.eo, self.lay, self.wts, self.y, self.ws, stream)

    def _capture(self):
        import torch

        s = torch.cuda.Stream(device=self.dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(2):
                self.dispatch()
                self.combine()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        gd, gc, gs = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd):
            self.dispatch()
        with torch.cuda.graph(gc):
            self.combine()
        with torch.cuda.graph(gs):  # the whole step: layout, dispatch, combine
            self.dispatch()
            self.combine()
        torch.cuda.synchronize()
        return gd, gc, gs

    def run_dispatch(self):
        if self.graphs:
            self.graphs[0].replay()
        else:
            self.dispatch()

    def run_combine(self):
        if self.graphs:
            self.graphs[1].replay()
        else:
            self.combine()

    def step_graph(self, n):
        """A CUDA graph of n whole steps back to back (cached per n)."""
        import torch

        if n not in self._step_graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(n):
                    self.dispatch()
                    self.combine()
            torch.cuda.synchronize()
            self._step_graphs[n] = g
        return self._step_graphs[n]

    def time_whole_steps(self, steps, warmup, flush=None, per_graph=1):
        """Per-step ms of whole steps (layout, dispatch and combine kernels) replayed
        back to back, `per_graph` steps per CUDA graph (a last, shorter graph makes the
        count exactly `steps`); eagerly the two calls per step.  `flush` (if given) runs
        before each step, outside the events, and implies one step per graph.  Returns
        one time per step (a graph's time divided among its steps)."""
        import torch

        if flush is not None or not self.graphs:
            per_graph = 1

        def run(n):
            if self.graphs:
                (self.graphs[2] if n == 1 else self.step_graph(n)).replay()
            else:
                for _ in range(n):
                    self.dispatch()
                    self.combine()

        sizes = [per_graph] * (steps // per_graph) + ([steps % per_graph] if steps % per_graph else [])
        for n in sorted(set(sizes)):  # capture (and warm) every graph before timing
            run(n)
        for _ in range(warmup):
            if flush is not None:
                flush()
            run(1)
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in sizes]
        for i, n in enumerate(sizes):
            if flush is not None:
                flush()
            evs[i][0].record()
            run(n)
            evs[i][1].record()
        torch.cuda.synchronize()
        out = []
        for e, n in zip(evs, sizes):
            out += [e[0].elapsed_time(e[1]) / n] * n
        return out

    def time_steps(self, steps, warmup, flush=None):
        """Per-step (dispatch ms, combine ms); `flush` (if given) runs before each step,
        outside the events."""
        import torch

        for _ in range(warmup):
            if flush is not None:
                flush()
            self.run_dispatch()
            self.run_combine()
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for i in range(steps):
            if flush is not None:
                flush()
            evs[i][0].record()
            self.run_dispatch()
            evs[i][1].record()
            self.run_combine()
            evs[i][2].record()
        torch.cuda.synchronize()
        return ([e[0].elapsed_time(e[1]) for e in evs], [e[1].elapsed_time(e[2]) for e in evs])


def time_low_latency(ep, w, dev, reps=200, per_graph=20):
    """LL dispatch / combine latency (L2 warm, as in decode):
    graph_replay_us -- one call per CUDA-graph replay, replays back to back
                       (launch-inclusive: includes the graph launch cost);
    gpu_us          -- per_graph calls captured in one graph (device time per call);
    eager_call_us   -- one eager call through the Python binding + synchronize
                       (host wall time)."""
    import numpy as np
    import torch

    T, H, K, E = w.num_tokens, w.hidden, w.num_topk, w.num_experts
    cap = w.num_max_tokens
    x = torch.from_numpy(w.x.view(np.int16)).to(dev).view(torch.bfloat16)
    idx = torch.from_numpy(w.topk_idx).to(dev)
    wts = torch.from_numpy(w.topk_weights).to(dev)
    rq = torch.empty((E, cap, H), dtype=torch.uint8, device=dev)
    rs = torch.empty((E, cap, H // 128), dtype=torch.float32, device=dev)
    cnt = torch.empty(E, dtype=torch.int32, device=dev)
    h = ep.LowLatencyHandle.empty(T, K, E, cap, dev)
    ws = torch.empty(ep.ep_workspace_bytes(1, E, 1), dtype=torch.uint8, device=dev)
    ep.ep_workspace_init(ws)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)

    def disp():
        ep.ep_low_latency_dispatch(x, idx, cap, E, rq, rs, cnt, h, ws)

    disp()
    torch.cuda.synchronize()
    q = rq.view(torch.float8_e4m3fn).to(torch.float32)
    eo = (q * rs.repeat_interleave(128, dim=-1)).to(torch.bfloat16)
    del q

    def comb():
        ep.ep_low_latency_combine(eo, h, wts, y, ws)

    def capture(fn, n):
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n):
                fn()
        for _ in range(5):
            g.replay()
        torch.cuda.synchronize()
        return g

    out = {}
    for name, fn in (("dispatch", disp), ("combine", comb)):
        g1 = capture(fn, 1)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        evs[0].record()
        for i in range(reps):
            g1.replay()
            evs[i + 1].record()
        torch.cuda.synchronize()
        replay_us = statistics.median(evs[i].elapsed_time(evs[i + 1]) * 1e3 for i in range(reps))
        gn = capture(fn, per_graph)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            gn.replay()
        e1.record()
        torch.cuda.synchronize()
        gpu_us = e0.elapsed_time(e1) * 1e3 / (10 * per_graph)
        walls = []
        for _ in range(50):
            t0 = time.perf_counter()
            fn()
            torch.cuda.synchronize()
            walls.append((time.perf_counter() - t0) * 1e6)
        out[name] = {"gpu_us": round(gpu_us, 2), "graph_replay_us": round(replay_us, 2),
                     "eager_call_us": round(statistics.median(walls), 2),
                     "tokens_per_s": round(T / (gpu_us * 1e-6))}
    if ep.ep_read_status(ws) != 0:
        raise RuntimeError("device status set in the low-latency run")
    out["config"] = f"{T} tokens x hidden {H}, top-{K} of {E} experts, capacity {cap}, FP8"

    # the peer-memory form: rank 0 of W = w.num_partitions sends the same batch into
    # the W owners' padded blocks [E/W, W*cap, H] (all on this GPU), and its combine
    # reads the rows back from them
    W = w.num_partitions
    epp = E // W
    owners = [dict(x=torch.empty((epp, W * cap, H), dtype=torch.uint8, device=dev),
                   s=torch.empty((epp, W * cap, H // 128), dtype=torch.float32, device=dev),
                   c=torch.empty((epp, W), dtype=torch.int32, device=dev),
                   eo=torch.empty((epp, W * cap, H), dtype=torch.bfloat16, device=dev))
              for _ in range(W)]
    tab = {k: torch.tensor([o[k].data_ptr() for o in owners], dtype=torch.int64, device=dev)
           for k in ("x", "s", "c", "eo")}
    for q, o in enumerate(owners):  # rank 0's block of each owner: the rows it would receive
        o["eo"][:, :cap] = eo[q * epp:(q + 1) * epp]

    def pdisp():
        ep.ep_peer_low_latency_dispatch(x, idx, cap, E, W, 0, tab["x"], tab["s"], tab["c"], h, ws)

    def pcomb():
        ep.ep_peer_low_latency_combine(tab["eo"], idx, h, wts, y, E, W, 0, ws)

    for name, fn in (("peer_dispatch", pdisp), ("peer_combine", pcomb)):
        gn = capture(fn, per_graph)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            gn.replay()
        e1.record()
        torch.cuda.synchronize()
        out[name] = {"gpu_us": round(e0.elapsed_time(e1) * 1e3 / (10 * per_graph), 2),
                     "ranks": W}
    if ep.ep_read_status(ws) != 0:
        raise RuntimeError("device status set in the peer low-latency run")
    del owners, tab
    return out


def time_epgroup(ep, w, dev, steps):
    """EpGroup(transport="peer") as whole calls through the Python API at one rank
    (workload w): dispatch = layout + count all-gather (NCCL) + plan + peer dispatch +
    receive barrier; combine = barrier + peer combine.  Per call: device time between
    CUDA events around the call (it includes any time the GPU waits for the host) and
    host time to return.  sync_sizes=True returns exact-size tensors, which needs the
    received counts on the host; sync_sizes=False keeps them on the device, and its
    whole steps are also timed launched back to back (step_us: device time per step;
    step_host_us: the host's time to issue one) and captured in a CUDA graph."""
    import socket

    import numpy as np
    import torch
    import torch.distributed as dist

    own = not dist.is_initialized()
    if own:
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    T, H, K, E = w.num_tokens, w.hidden, w.num_topk, w.num_experts
    g = ep.EpGroup(E, transport="peer", hidden=H, max_tokens=T, num_topk=K,
                   capacity=T * K + 16, device=dev)
    out = {"ranks": 1, "tokens": T}
    try:
        x = torch.from_numpy(w.x.view(np.int16)).to(dev).view(torch.bfloat16)
        idx = torch.from_numpy(w.topk_idx).to(dev)
        wts = torch.from_numpy(w.topk_weights).to(dev)
        for sync in (True, False):
            rec = {}
            d_dev, d_host, c_dev, c_host = [], [], [], []
            for i in range(steps + 3):
                e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                e[0].record()
                t0 = time.perf_counter()
                res = g.dispatch(x, idx, wts, sync_sizes=sync)
                t1 = time.perf_counter()
                e[1].record()
                ctx = res[4]
                t2 = time.perf_counter()
                g.combine(g.expert_out_buffer(ctx), ctx, wts)
                t3 = time.perf_counter()
                e[2].record()
                torch.cuda.synchronize()
                if i >= 3:
                    d_dev.append(e[0].elapsed_time(e[1]) * 1e3)
                    c_dev.append(e[1].elapsed_time(e[2]) * 1e3)
                    d_host.append((t1 - t0) * 1e6)
                    c_host.append((t3 - t2) * 1e6)
            rec["dispatch_us"] = round(statistics.median(d_dev), 2)
            rec["dispatch_call_host_us"] = round(statistics.median(d_host), 1)
            rec["combine_us"] = round(statistics.median(c_dev), 2)
            rec["combine_call_host_us"] = round(statistics.median(c_host), 1)
            if not sync:
                # whole steps launched back to back, as a training loop does: the host
                # runs ahead of the device unless its calls take longer than the kernels
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record()
                t0 = time.perf_counter()
                for _ in range(steps):
                    res = g.dispatch(x, idx, wts, sync_sizes=False)
                    g.combine(g.expert_out_buffer(res[4]), res[4], wts)
                t1 = time.perf_counter()
                e[1].record()
                torch.cuda.synchronize()
                rec["step_us"] = round(e[0].elapsed_time(e[1]) * 1e3 / steps, 2)
                rec["step_host_us"] = round((t1 - t0) * 1e6 / steps, 1)
            out["sync_sizes" if sync else "no_sync"] = rec
        # with sync_sizes=False nothing in a step waits on the host, so the whole step
        # (NCCL collectives included) can be captured in a CUDA graph and replayed
        try:
            cs = torch.cuda.Stream(device=dev)
            cs.wait_stream(torch.cuda.current_stream())

            def step():
                res = g.dispatch(x, idx, wts, sync_sizes=False)
                g.combine(g.expert_out_buffer(res[4]), res[4], wts)

            with torch.cuda.stream(cs):
                step()
                step()
            torch.cuda.current_stream().wait_stream(cs)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=cs):
                step()
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                graph.replay()
            e1.record()
            torch.cuda.synchronize()
            out["no_sync_graph_step_us"] = round(e0.elapsed_time(e1) * 1e3 / steps, 2)
            del graph
        except Exception as exc:  # report, do not hide
            out["no_sync_graph_error"] = repr(exc)
        if ep.ep_read_status(g.workspace) != 0:
            raise RuntimeError("device status set in the EpGroup run")
    finally:
        g.close()
        if own:
            dist.destroy_process_group()
    out["note"] = ("one rank: the owner's buffers are this GPU's, so no NVLink traffic; "
                   "the expert outputs are whatever the buffer holds (the time does not "
                   "depend on them)")
    return out


def time_layout_alone(ep, runner, per_graph=20, reps=10):
    """The layout call by itself (ep_get_dispatch_layout on the runner's routing, with a
    handle and workspace of its own): per_graph calls captured in one CUDA graph,
    replayed back to back; device time per call.  In the benchmark step the layout
    is followed by the dispatch kernel, which starts loading and quantising during it."""
    import torch

    lay = ep.Layout.empty(runner.T, runner.K, runner.E, runner.P, runner.dev)
    ws = torch.empty(ep.ep_workspace_bytes(runner.T, runner.E, runner.P), dtype=torch.uint8,
                     device=runner.dev)
    ep.ep_workspace_init(ws)

    def call():
        ep.ep_get_dispatch_layout(runner.idx, runner.E, runner.P, lay, ws)

    s = torch.cuda.Stream(device=runner.dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()
        call()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(per_graph):
            call()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    if ep.ep_read_status(ws) != 0:
        raise RuntimeError("device status set in the layout run")
    return e0.elapsed_time(e1) * 1e3 / (reps * per_graph)


def time_backward(ep, runner, steps):
    """Backward pair on the runner's workload: ep_dispatch_backward (row gradients ->
    grad_x, weight-gradient gather) and ep_combine_backward (grad_y -> expert-row
    gradients and weight gradients), each captured as a CUDA graph, back to back."""
    import torch

    T, H, K, R = runner.T, runner.H, runner.K, runner.R
    dev = runner.x.device
    g_rows = runner.eo  # any BF16 [rows, H] buffer serves as the row gradients
    grw = torch.randn(max(R, 1), device=dev)
    gx = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    gw1 = torch.empty((T, K), dtype=torch.float32, device=dev)
    gy = torch.randn((T, H), device=dev).to(torch.bfloat16)
    geo = torch.empty_like(runner.eo)
    gw2 = torch.empty((T, K), dtype=torch.float32, device=dev)

    def dbwd():
        ep.ep_dispatch_backward(g_rows, runner.lay, gx, runner.ws, grw, gw1)

    def cbwd():
        ep.ep_combine_backward(gy, runner.eo, runner.lay, runner.wts, geo, gw2, runner.ws)

    out = {}
    bytes_d = R * H * 2 + T * H * 2 + T * K * 4 + R * 4 + T * K * 4
    bytes_c = T * H * 2 + R * H * 2 * 2 + T * K * 8 + T * K * 4
    for name, fn, nbytes in (("dispatch_backward", dbwd, bytes_d),
                             ("combine_backward", cbwd, bytes_c)):
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        evs[0].record()
        for i in range(steps):
            g.replay()
            evs[i + 1].record()
        torch.cuda.synchronize()
        us = statistics.mean(evs[i].elapsed_time(evs[i + 1]) for i in range(steps)) * 1e3
        out[name] = {"us": round(us, 2), "bytes": nbytes, "gbs": round(nbytes / (us * 1e-6) / 1e9, 1)}
    if ep.ep_read_status(runner.ws) != 0:
        raise RuntimeError("device status set in the backward run")
    return out


def time_lb(ep, dev, steps, seed, scale=1):
    """Redundant experts on the stress workload's 288-slot map (32 replicas of the
    hottest experts): weight prefetch with one FP8 expert per slot (gate, up and
    down projections, 3 x 7168 x 2048 bytes) and the fp32 gradient reduce over
    one 7168 x 2048 matrix per slot, each captured as a CUDA graph."""
    import numpy as np
    import torch
    from workloads import make_workload

    po = make_workload("stress", seed=seed, num_tokens=64, hidden=128).meta["primary_of"]
    S = po.size
    groups = np.bincount(po, minlength=S)
    replicas = int((po != np.arange(S)).sum())
    in_groups = int(groups[po][groups[po] > 1].size)  # slots whose group has > 1 member
    nbytes = 3 * 7168 * 2048 // scale // 16 * 16
    n = 7168 * 2048 // scale // 4 * 4
    dpo = torch.from_numpy(po).to(dev)
    weights = torch.empty((S, nbytes), dtype=torch.uint8, device=dev)
    grads = torch.zeros((S, n), dtype=torch.float32, device=dev)
    ws = torch.empty(ep.ep_workspace_bytes(1, 1, 1), dtype=torch.uint8, device=dev)
    ep.ep_workspace_init(ws)
    out = {"slots": S, "replicas": replicas, "bytes_per_slot": nbytes, "grad_floats_per_slot": n}
    cases = (("prefetch_weights", lambda: ep.ep_lb_prefetch_weights(dpo, weights, ws),
              2 * replicas * nbytes),
             ("reduce_grads", lambda: ep.ep_lb_reduce_grads(dpo, grads, ws), 2 * in_groups * n * 4))
    for name, fn, nb in cases:
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        evs[0].record()
        for i in range(steps):
            g.replay()
            evs[i + 1].record()
        torch.cuda.synchronize()
        us = statistics.mean(evs[i].elapsed_time(evs[i + 1]) for i in range(steps)) * 1e3
        out[name] = {"us": round(us, 2), "bytes": nb, "gbs": round(nb / (us * 1e-6) / 1e9, 1)}
    if ep.ep_read_status(ws) != 0:
        raise RuntimeError("device status set in the redundant-expert run")
    del weights, grads
    torch.cuda.empty_cache()
    return out


def time_dedup(ep, w, dev, steps):
    """Deduplicated dispatch (one row per token and partition) and its combine on
    workload w, each captured as a CUDA graph; the partition outputs come from a
    partition-local identity stand-in computed once."""
    import numpy as np
    import torch

    T, H, K, E, P = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
    fp8 = w.quant == "fp8"
    rows = max(T * min(P, K), 1)
    x = torch.from_numpy(w.x.view(np.int16)).to(dev).view(torch.bfloat16)
    idx = torch.from_numpy(w.topk_idx).to(dev)
    wts = torch.from_numpy(w.topk_weights).to(dev)
    rq = torch.empty((rows, H), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
    rs = torch.empty((rows, H // 128), dtype=torch.float32, device=dev) if fp8 else None
    ri = torch.empty((rows, K), dtype=torch.int32, device=dev)
    rw = torch.empty((rows, K), dtype=torch.float32, device=dev)
    lay = ep.Layout.empty(T, P, P, P, dev)
    ws = torch.empty(ep.ep_workspace_bytes(T, E, P), dtype=torch.uint8, device=dev)
    ep.ep_workspace_init(ws)
    quant = ep.EP_QUANT_FP8_E4M3_1X128 if fp8 else ep.EP_QUANT_NONE

    def disp():
        ep.ep_dispatch_dedup(x, idx, wts, E, P, quant, rq, rs, ri, rw, lay, ws)

    disp()
    torch.cuda.synchronize()
    R = int(lay.num_recv.item())
    v = (rq.view(torch.float8_e4m3fn).to(torch.float32) * rs.repeat_interleave(128, dim=1)) \
        if fp8 else rq.to(torch.float32)
    part = (v * torch.where(ri >= 0, rw, 0).sum(dim=1, keepdim=True)).to(torch.bfloat16)
    del v
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)

    def comb():
        ep.ep_combine_dedup(part[:max(R, 1)], lay, y, ws)

    payload = R * H * (1 if fp8 else 2) + (R * (H // 128) * 4 if fp8 else 0)
    bytes_d = (T * H * 2 + payload + T * K * 12 + R * K * 8 + R * 4 + T * P * 4
               + (P + 1) * 4 + 2 * P * 4 + T * P)
    bytes_c = R * H * 2 + T * H * 2 + T * P * 4
    out = {"rows": R, "rows_per_expert_path": int((w.topk_idx >= 0).sum())}
    for name, fn, nbytes in (("dispatch", disp, bytes_d), ("combine", comb, bytes_c)):
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        evs[0].record()
        for i in range(steps):
            g.replay()
            evs[i + 1].record()
        torch.cuda.synchronize()
        us = statistics.mean(evs[i].elapsed_time(evs[i + 1]) for i in range(steps)) * 1e3
        out[name + "_us"] = round(us, 2)
        out[name + "_gbs"] = round(nbytes / (us * 1e-6) / 1e9, 1)
    if ep.ep_read_status(ws) != 0:
        raise RuntimeError("device status set in the deduplicated run")
    return out


def time_peer(ep, w, dev, steps):
    """The peer-memory (multi-GPU) kernels on workload w with every owner's buffers on
    this GPU: rank 0 of W = w.num_partitions holds all tokens, the other ranks none.
    Dispatch = layout + the count copy that stands for the all-gather + plan + peer
    dispatch (rows stored into the W owners' buffers); combine = peer combine (rows
    loaded from them).  Same algorithmic bytes as the one-GPU step; the stores and
    loads stay in this GPU's HBM, so this measures the kernels, not NVLink.  Then
    the same for deduplicated rows (one per token and owner rank)."""
    import numpy as np
    import torch

    T, H, K, E, W = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
    fp8 = w.quant == "fp8"
    epp = E // W
    x = torch.from_numpy(w.x.view(np.int16)).to(dev).view(torch.bfloat16)
    idx = torch.from_numpy(w.topk_idx).to(dev)
    wts = torch.from_numpy(w.topk_weights).to(dev)
    lay = ep.Layout.empty(T, K, E, W, dev)
    ws = torch.empty(ep.ep_workspace_bytes(T, E, W), dtype=torch.uint8, device=dev)
    ep.ep_workspace_init(ws)
    ep.ep_get_dispatch_layout(idx, E, W, lay, ws)
    torch.cuda.synchronize()
    per_part = lay.num_tokens_per_expert.view(W, epp).sum(dim=1)
    cap = int(per_part.max().item()) + 16
    R = int(lay.num_recv.item())
    bufs = [dict(x=torch.empty((cap, H), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev),
                 s=torch.empty((cap, H // 128), dtype=torch.float32, device=dev),
                 i=torch.empty(cap, dtype=torch.int32, device=dev),
                 w=torch.empty(cap, dtype=torch.float32, device=dev),
                 eo=torch.empty((cap, H), dtype=torch.bfloat16, device=dev)) for _ in range(W)]
    tables = ep.PeerTables.from_addresses(dev, cap, *[[b[k].data_ptr() for b in bufs]
                                                      for k in ("x", "s", "i", "w", "eo")])
    counts = torch.zeros((W, E), dtype=torch.int32, device=dev)
    dst = torch.empty(E, dtype=torch.int32, device=dev)
    rc = torch.empty(epp, dtype=torch.int32, device=dev)
    ro = torch.empty(epp + 1, dtype=torch.int32, device=dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    quant = ep.EP_QUANT_FP8_E4M3_1X128 if fp8 else ep.EP_QUANT_NONE

    def disp():
        ep.ep_get_dispatch_layout(idx, E, W, lay, ws)
        counts[0].copy_(lay.num_tokens_per_expert)  # stands for the all-gather
        ep.ep_peer_plan(counts, 0, lay.expert_offset, cap, dst, rc, ro, ws)
        ep.ep_peer_dispatch(x, idx, wts, E, W, quant, lay, dst, tables, ws)

    def comb():
        ep.ep_peer_combine(tables, lay, idx, dst, wts, y, E, W, ws)

    disp()
    torch.cuda.synchronize()
    for b, n in zip(bufs, per_part.tolist()):  # identity experts on the received rows
        if fp8:
            v = b["x"][:n].view(torch.float8_e4m3fn).to(torch.float32)
            b["eo"][:n] = (v * b["s"][:n].repeat_interleave(128, dim=1)).to(torch.bfloat16)
        else:
            b["eo"][:n] = b["x"][:n]
    bytes_d, bytes_c = algorithmic_bytes(T, H, K, E, W, R, fp8)
    out = {"ranks": W, "tokens": T, "recv_rows": R, "capacity": cap}
    for name, fn, nbytes in (("dispatch", disp, bytes_d), ("combine", comb, bytes_c)):
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        evs[0].record()
        for i in range(steps):
            g.replay()
            evs[i + 1].record()
        torch.cuda.synchronize()
        us = statistics.mean(evs[i].elapsed_time(evs[i + 1]) for i in range(steps)) * 1e3
        out[name + "_us"] = round(us, 2)
        out[name + "_gbs"] = round(nbytes / (us * 1e-6) / 1e9, 1)
    # deduplicated rows: one per (token, owner rank), [K] id / weight lists
    dlay = ep.Layout.empty(T, W, W, W, dev)
    ep.ep_get_dispatch_layout_dedup(idx, E, W, dlay, ws)
    torch.cuda.synchronize()
    dper = dlay.num_tokens_per_expert.clone()
    dcap = int(dper.max().item()) + 16
    Rd = int(dlay.num_recv.item())
    dbufs = [dict(x=b["x"], s=b["s"], eo=b["eo"],
                  i=torch.empty((dcap, K), dtype=torch.int32, device=dev),
                  w=torch.empty((dcap, K), dtype=torch.float32, device=dev)) for b in bufs]
    assert dcap <= cap
    dtables = ep.PeerTables.from_addresses(dev, dcap, *[[b[k].data_ptr() for b in dbufs]
                                                        for k in ("x", "s", "i", "w", "eo")])
    dcounts = torch.zeros((W, W), dtype=torch.int32, device=dev)
    ddst = torch.empty(W, dtype=torch.int32, device=dev)
    drc = torch.empty(1, dtype=torch.int32, device=dev)
    dro = torch.empty(2, dtype=torch.int32, device=dev)

    def ddisp():
        ep.ep_get_dispatch_layout_dedup(idx, E, W, dlay, ws)
        dcounts[0].copy_(dlay.num_tokens_per_expert)  # stands for the all-gather
        ep.ep_peer_plan(dcounts, 0, dlay.expert_offset, dcap, ddst, drc, dro, ws)
        ep.ep_peer_dispatch_dedup(x, idx, wts, E, W, quant, dlay, ddst, dtables, ws)

    def dcomb():
        ep.ep_peer_combine_dedup(dtables, dlay, ddst, y, W, ws)

    payload = Rd * H * (1 if fp8 else 2) + (Rd * (H // 128) * 4 if fp8 else 0)
    bytes_dd = (T * H * 2 + payload + T * K * 12 + Rd * K * 8 + Rd * 4 + T * W * 4
                + (W + 1) * 4 + 2 * W * 4 + T * W)
    bytes_dc = Rd * H * 2 + T * H * 2 + T * W * 4
    out["dedup_rows"] = Rd
    for name, fn, nbytes in (("dedup_dispatch", ddisp, bytes_dd), ("dedup_combine", dcomb, bytes_dc)):
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        evs[0].record()
        for i in range(steps):
            g.replay()
            evs[i + 1].record()
        torch.cuda.synchronize()
        us = statistics.mean(evs[i].elapsed_time(evs[i + 1]) for i in range(steps)) * 1e3
        out[name + "_us"] = round(us, 2)
        out[name + "_gbs"] = round(nbytes / (us * 1e-6) / 1e9, 1)
    if ep.ep_read_status(ws) != 0:
        raise RuntimeError("device status set in the peer-memory run")
    del bufs, tables, dbufs, dtables
    torch.cuda.empty_cache()
    return out


def time_e2e(ep, runner, steps):
    """The same step through the public API with host buffers, pipelined the way a
    serving loop would run it: every step copies its inputs (x, topk_idx,
    topk_weights) from pinned host memory on a copy-in stream, runs dispatch +
    combine on a compute stream, and copies y back to pinned host memory on a
    copy-out stream; inputs and outputs are double-buffered so step i's copies
    overlap step i-1's kernels.  Timed with CUDA events from before the first copy
    to after the last copy-back (device time over all steps)."""
    import torch

    dev = runner.x.device
    hx = [runner.x.cpu().pin_memory() for _ in range(2)]
    hi = [runner.idx.cpu().pin_memory() for _ in range(2)]
    hw = [runner.wts.cpu().pin_memory() for _ in range(2)]
    hy = [torch.empty(runner.y.shape, dtype=runner.y.dtype).pin_memory() for _ in range(2)]
    dx = [runner.x, runner.x.clone()]
    di = [runner.idx, runner.idx.clone()]
    dw = [runner.wts, runner.wts.clone()]
    dy = [runner.y, torch.empty_like(runner.y)]
    h2d = hx[0].numel() * 2 + hi[0].numel() * 8 + hw[0].numel() * 4
    d2h = hy[0].numel() * 2
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [ev(), ev()]     # inputs of buffer b copied
    cmp_done = [ev(), ev()]    # kernels that read/write buffer b finished
    out_done = [ev(), ev()]    # y of buffer b copied back
    for b in range(2):
        for e in (cmp_done[b], out_done[b]):
            e.record(s_cmp)

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(cmp_done[b])        # the kernels of step i-2 are done with dx[b]
            dx[b].copy_(hx[b], non_blocking=True)
            di[b].copy_(hi[b], non_blocking=True)
            dw[b].copy_(hw[b], non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_done[b])
            s_cmp.wait_event(out_done[b])       # y of step i-2 has been copied out
            ep.ep_dispatch(dx[b], di[b], dw[b], runner.E, runner.P, runner.quant, runner.recv_q,
                           runner.recv_s, runner.recv_i, runner.recv_w, runner.lay, runner.ws,
                           s_cmp)
            ep.ep_combine(runner.eo, runner.lay, dw[b], dy[b], runner.ws, s_cmp)
            cmp_done[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[b])
            hy[b].copy_(dy[b], non_blocking=True)
            out_done[b].record(s_out)

    for i in range(4):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        step(i)
    s_in.wait_stream(s_out)
    s_in.wait_stream(s_cmp)
    t1.record(s_in)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return ms, h2d, d2h


def host_cores():
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class ShardedOracle:
    """The oracle, unchanged, on the host's cores: the layout of the batch runs
    serially (every row depends on all tokens), then dispatch and combine run over
    contiguous token shards, one per thread (the oracle is C behind ctypes, which
    releases the GIL for each call).  A shard's dispatch lays out and quantises its
    own tokens (the same per-token work as in the whole batch; the rows land in a
    shard-local buffer); the combine of a shard reads the batch's expert outputs
    through the batch's layout."""

    def __init__(self, w, threads):
        import concurrent.futures
        import oracle

        self.oracle, self.w = oracle, w
        self.threads = max(1, threads)
        T = w.num_tokens
        bounds = [T * i // self.threads for i in range(self.threads + 1)]
        self.shards = [(a, b) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
        self.pool = concurrent.futures.ThreadPoolExecutor(max_workers=self.threads)
        d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, w.num_experts, w.num_partitions,
                            quant=w.quant)
        self.R = int(d["num_recv"][0])
        self.eo = oracle.identity_expert(d["recv_x"], d["recv_scales"], quant=w.quant)

    def one_pass(self):
        """(layout s, dispatch s, combine s) of one pass over the batch."""
        o, w = self.oracle, self.w
        E, P = w.num_experts, w.num_partitions
        t0 = time.perf_counter()
        lay = o.layout(w.topk_idx, E, P)
        t1 = time.perf_counter()
        list(self.pool.map(lambda ab: o.dispatch(w.x[ab[0]:ab[1]], w.topk_idx[ab[0]:ab[1]],
                                                 w.topk_weights[ab[0]:ab[1]], E, P,
                                                 quant=w.quant), self.shards))
        t2 = time.perf_counter()
        list(self.pool.map(lambda ab: o.combine(self.eo, lay["row_of"][ab[0]:ab[1]],
                                                w.topk_weights[ab[0]:ab[1]]), self.shards))
        t3 = time.perf_counter()
        return t1 - t0, t2 - t1, t3 - t2

    def close(self):
        self.pool.shutdown()


def cpu_baseline(w, min_seconds=10.0, configs=True):
    """The oracle, as it stands, on the same batch: single-threaded C (the reported
    value), then the same work spread over the host's cores, and per-workload
    layout / dispatch / combine medians of the spread-out form."""
    import oracle
    from workloads import make_workload

    T, H, K, E, P = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
    d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, E, P, quant=w.quant)
    eo = oracle.identity_expert(d["recv_x"], d["recv_scales"], quant=w.quant)
    bd, bc = algorithmic_bytes(T, H, K, E, P, int(d["num_recv"][0]), w.quant == "fp8")
    passes, t = 0, 0.0
    while t < min_seconds and passes < 50:
        t0 = time.perf_counter()
        dd = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, E, P, quant=w.quant)
        oracle.combine(eo, dd["row_of"], w.topk_weights)
        t += time.perf_counter() - t0
        passes += 1
    cores = host_cores()
    out = {"value": round((bd + bc) * passes / t / 1e9, 3), "unit": "GB/s", "cores": 1,
           "kind": "oracle", "host_cores": cores,
           "sample": f"the full {T}-token batch (layout + dispatch + combine), {passes} passes, "
                     f"{t:.1f} s, single-threaded C"}
    so = ShardedOracle(w, cores)
    try:
        so.one_pass()
        runs = [so.one_pass() for _ in range(5)]
    finally:
        so.close()
    tt = statistics.median([sum(r) for r in runs])
    out["threaded"] = {
        "value": round((bd + bc) / tt / 1e9, 3), "unit": "GB/s", "cores": so.threads,
        "ms_per_step": round(tt * 1e3, 2),
        "sample": f"the full {T}-token batch, median of 5 passes: layout serial, dispatch and "
                  f"combine over {len(so.shards)} token shards in {so.threads} threads"}
    if configs:
        per = {}
        try:  # the low-latency batch through the oracle's padded layout, one thread
            wl = make_workload("ll", seed=w.seed)
            dl = oracle.ll_dispatch(wl.x, wl.topk_idx, wl.num_experts, wl.num_max_tokens)
            eol = oracle.identity_expert(
                dl["recv_x"].reshape(-1, wl.hidden),
                dl["recv_scales"].reshape(-1, wl.hidden // 128)).reshape(
                    wl.num_experts, wl.num_max_tokens, wl.hidden)
            rl = []
            for _ in range(4):
                t0 = time.perf_counter()
                oracle.ll_dispatch(wl.x, wl.topk_idx, wl.num_experts, wl.num_max_tokens)
                t1 = time.perf_counter()
                oracle.ll_combine(eol, dl["ll_row_of"], wl.topk_weights)
                rl.append((t1 - t0, time.perf_counter() - t1))
            dm, cm = (statistics.median(r[i] for r in rl[1:]) for i in range(2))
            per["ll"] = {"tokens": wl.num_tokens, "dispatch_ms": round(dm * 1e3, 3),
                         "combine_ms": round(cm * 1e3, 3),
                         "dispatch_tokens_per_s": round(wl.num_tokens / dm),
                         "combine_tokens_per_s": round(wl.num_tokens / cm),
                         "sample": "padded low-latency layout (layout fused into the dispatch), "
                                   "single-threaded, median of 3 passes"}
        except Exception as exc:  # report, do not hide
            per["ll"] = {"error": repr(exc)}
        for name in ("normal", "skew", "bf16", "stress"):
            try:
                n = 4096 if name == "stress" else None  # a bounded sample of the largest batch
                wx = make_workload(name, seed=w.seed, num_tokens=n)
                sx = ShardedOracle(wx, cores)
                try:
                    sx.one_pass()
                    rr = [sx.one_pass() for _ in range(3)]
                finally:
                    sx.close()
                lm, dm, cm = (statistics.median(r[i] for r in rr) for i in range(3))
                per[name] = {"tokens": wx.num_tokens, "layout_ms": round(lm * 1e3, 3),
                             "dispatch_ms": round(dm * 1e3, 3), "combine_ms": round(cm * 1e3, 3),
                             "dispatch_tokens_per_s": round(wx.num_tokens / (lm + dm)),
                             "combine_tokens_per_s": round(wx.num_tokens / cm)}
                if n is not None:
                    per[name]["sample"] = f"the stress recipe drawn at {n} tokens"
            except Exception as exc:  # report, do not hide
                per[name] = {"error": repr(exc)}
        out["configs"] = per
        out["configs_note"] = (f"oracle over {cores} threads (layout serial, dispatch and combine "
                               "sharded over tokens), medians of 3 passes; dispatch tokens/s "
                               "includes the layout")
    return out


L2_TEXT = ("inputs larger than L2: each step reads 529 MB (x + expert outputs) and writes "
           "294 MB, steps back to back, no flush")


def workload_config(name, w, R, step_bytes, seed, world, l2_flush="none"):
    """The `config` object of the JSON line: what the workload is, identical in
    both arms for the same workload and seed."""
    return {
        "workload": WORKLOAD_TEXT[name],
        "tokens_per_gpu": w.num_tokens, "hidden": w.hidden, "topk": w.num_topk,
        "experts": w.num_experts, "partitions": w.num_partitions, "recv_rows": R,
        "bytes_per_step": step_bytes, "seed": seed,
        "l2": L2_TEXT if l2_flush == "none"
        else f"flushed before every step by a 256 MiB {l2_flush} (outside the events)",
        "parallelism": f"replicas x{world} (independent batches, no exchange)",
    }


def make_flush(mode, dev):
    """L2 flush before a step: write (zero) or read (sum) a 256 MiB buffer."""
    import torch

    if mode == "none":
        return None
    buf = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    if mode == "write":
        return lambda: buf.zero_()
    return lambda: buf.sum()


def reduce_max_over_ranks(values, world, device):
    """Element-wise max of per-rank float values across the process group."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def run_ours(args):
    import torch
    import torch.distributed as dist

    import combine_get_dispatch_05_b200 as ep
    from workloads import make_workload

    rank, world, local = env_rank()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    sampler = ClockSampler(local)
    sampler.start()
    w = make_workload(args.workload, seed=args.seed + rank)
    runner = PathRunner(ep, w, dev, use_graphs=not args.eager)
    flush = make_flush(args.l2_flush, dev)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    s_ms = runner.time_whole_steps(args.steps, args.warmup, flush, per_graph=args.steps_per_graph)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t1 = time.time()
    sampler.mark(t0, t1)
    # breakdown: the same steps again with the dispatch and the combine launched as two
    # graphs, events between them (the boundary costs the step a few us); and the
    # whole step as one graph per step, for reference
    d_ms, c_ms = runner.time_steps(args.steps, 3, flush)
    one_ms = runner.time_whole_steps(args.steps, 3, flush, per_graph=1)
    layout_us = time_layout_alone(ep, runner)
    torch.cuda.synchronize()
    status = ep.ep_read_status(runner.ws)

    tot = reduce_max_over_ranks([sum(s_ms), sum(c_ms), sum(d_ms), sum(one_ms), layout_us],
                                world, dev)
    layout_us = tot[4]
    total_ms = tot[0]
    ms_step = total_ms / args.steps
    step_bytes = runner.bytes_dispatch + runner.bytes_combine
    value = world * step_bytes / (ms_step * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        e_ms, h2d, d2h = time_e2e(ep, runner, max(5, min(args.steps, 50)))
        e_ms = reduce_max_over_ranks([e_ms], world, dev)[0]  # the slowest rank's time
        e2e = {"value": round(world * step_bytes / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
               "ms_per_step": round(e_ms, 4), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "path": "ep_dispatch + ep_combine (Python binding -> C ABI), pinned host buffers, "
                       "copy-in / compute / copy-out streams, double-buffered"}
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peak, peak_kind = measured_peaks()
    comb_us = tot[1] / args.steps * 1e3
    disp_us = tot[2] / args.steps * 1e3
    comb_gbs = runner.bytes_combine / (comb_us * 1e-6) / 1e9
    disp_gbs = runner.bytes_dispatch / (disp_us * 1e-6) / 1e9
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE_TEXT[runner.fp8],
        "data": "synthetic",
        "config": workload_config(args.workload, w, runner.R, step_bytes, args.seed, world,
                                  args.l2_flush),
        "launch": (f"CUDA graphs of {min(args.steps_per_graph, args.steps)} whole steps each "
                   "(layout, dispatch as a programmatic dependent of the layout, combine; the next "
                   "step's layout a programmatic dependent of the combine), replayed back to back; "
                   "one graph per step: %.2f us per step" % (tot[3] / args.steps * 1e3))
        if not args.eager and args.l2_flush == "none" else
        ("one CUDA graph per step (L2 flushed between steps)" if not args.eager else "eager"),
        "breakdown_note": "dispatch and combine intervals from a second pass of the same steps "
                          "with the two calls captured as separate graphs and events between "
                          "them; their sum exceeds the whole-step time by the graph boundary",
        "breakdown": {
            "layout": {"us": round(layout_us, 2),
                       "note": "the layout call alone, 20 calls per CUDA graph back to back; "
                               "inside the dispatch interval below it overlaps the dispatch "
                               "kernel's loads"},
            "dispatch": {"us": round(disp_us, 2), "bytes": runner.bytes_dispatch,
                         "gbs": round(disp_gbs, 1), "frac": round(disp_gbs / peak, 4),
                         "tokens_per_s": round(w.num_tokens / (disp_us * 1e-6)),
                         "kernels": "layout (cooperative) + dispatch_%s (programmatic dependent "
                                    "launch)" % ("fp8" if runner.fp8 else "bf16"),
                         "traffic": {
                             "layout_kernel": profiled_traffic(
                                 "layout_kernel_normal_4096x7168.md", LAYOUT_SOURCES),
                             "dispatch_fp8_kernel": profiled_traffic(
                                 "dispatch_fp8_kernel_normal_4096x7168.md", DISPATCH_SOURCES)}
                         if args.workload == "normal" and runner.fp8 else None},
            "combine": {"us": round(comb_us, 2), "bytes": runner.bytes_combine,
                        "gbs": round(comb_gbs, 1), "frac": round(comb_gbs / peak, 4),
                        "tokens_per_s": round(w.num_tokens / (comb_us * 1e-6)),
                        "kernels": "combine"},
        },
        "roofline": {
            "bound": "hbm", "kernel": "combine_kernel", "achieved": round(comb_gbs, 1),
            "peak": peak, "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
            if peak_kind == "measured" else "fallback 6.65 TB/s",
            "unit": "GB/s", "frac": round(comb_gbs / peak, 4),
            "traffic": profiled_traffic("combine_kernel_normal_4096x7168.md", COMBINE_SOURCES)
            if args.workload == "normal" else None,
        },
        "gpu_launches": 3 * args.steps,
        "device_status": status,
        "clocks": clocks,
    }
    if e2e is not None:
        result["e2e"] = e2e
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        result["cpu_baseline"] = cpu_baseline(w)
    if not args.no_extra:
        extra = {}
        want = set(args.extras.split(",")) if args.extras else None

        def workload_row(name):
            wx = make_workload(name, seed=args.seed)
            r = PathRunner(ep, wx, dev, use_graphs=not args.eager)
            ss = r.time_whole_steps(args.extra_steps, 3, flush, per_graph=args.steps_per_graph)
            dd, cc = r.time_steps(args.extra_steps, 3, flush)
            du, cu = statistics.mean(dd) * 1e3, statistics.mean(cc) * 1e3
            su = statistics.mean(ss) * 1e3
            row = {
                "tokens": wx.num_tokens, "hidden": wx.hidden, "topk": wx.num_topk,
                "experts": wx.num_experts, "partitions": wx.num_partitions,
                "quant": wx.quant, "recv_rows": r.R,
                "dispatch_us": round(du, 2),
                "dispatch_gbs": round(r.bytes_dispatch / (du * 1e-6) / 1e9, 1),
                "dispatch_tokens_per_s": round(wx.num_tokens / (du * 1e-6)),
                "combine_us": round(cu, 2),
                "combine_gbs": round(r.bytes_combine / (cu * 1e-6) / 1e9, 1),
                "combine_tokens_per_s": round(wx.num_tokens / (cu * 1e-6)),
                "step_us": round(su, 2),
                "step_gbs": round((r.bytes_dispatch + r.bytes_combine) / (su * 1e-6) / 1e9, 1),
                "status": ep.ep_read_status(r.ws)}
            del r
            torch.cuda.empty_cache()
            return row

        def on_workload(fn):
            def run():
                out = fn()
                out["workload"] = args.workload
                return out
            return run

        jobs = [
            ("backward", on_workload(lambda: time_backward(ep, runner, args.extra_steps))),
            ("dedup", on_workload(lambda: time_dedup(ep, w, dev, args.extra_steps))),
            ("peer", on_workload(lambda: time_peer(ep, w, dev, args.extra_steps))),
            # a group of one rank; with more ranks the group would span GPUs
            ("epgroup", on_workload(lambda: time_epgroup(ep, w, dev, min(args.extra_steps, 20))))
            if world == 1 else None,
            ("lb", lambda: time_lb(ep, dev, min(args.extra_steps, 20), args.seed, args.lb_scale)),
            ("ll", lambda: time_low_latency(ep, make_workload("ll", seed=args.seed), dev)),
        ] + [(name, lambda name=name: workload_row(name)) for name in ("skew", "bf16", "stress")]
        for job in jobs:
            if job is None or (want is not None and job[0] not in want):
                continue
            try:
                extra[job[0]] = job[1]()
            except Exception as exc:  # report, do not hide
                extra[job[0]] = {"error": repr(exc)}
        result["configs"] = extra
    print(json.dumps(result), flush=True)


# -------------------------------------------------------- reference arm -----

def token_prefix(w, n):
    """The first n tokens of a workload (a bounded sample of it)."""
    import dataclasses

    if n >= w.num_tokens:
        return w
    return dataclasses.replace(w, num_tokens=n, x=w.x[:n], topk_idx=w.topk_idx[:n],
                               topk_weights=w.topk_weights[:n])


def run_reference(args):
    """The CPU oracle as it stands, on the host's cores (layout serial, dispatch and
    combine over token shards), on the same workload or a bounded prefix of it."""
    rank, world, _ = env_rank()
    if rank != 0:
        return
    import oracle
    from workloads import make_workload

    w = make_workload(args.workload, seed=args.seed)
    T, H, K, E, P = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
    fp8 = w.quant == "fp8"
    R_full = int(oracle.layout(w.topk_idx, E, P)["num_recv"][0])
    bd_full, bc_full = algorithmic_bytes(T, H, K, E, P, R_full, fp8)
    cores = host_cores()

    # calibrate seconds per token, then size each step's sample so the whole run
    # stays near two minutes
    n_cal = min(T, 256)
    cal = ShardedOracle(token_prefix(w, n_cal), cores)
    try:
        cal.one_pass()
        per_tok = sum(cal.one_pass()) / n_cal
    finally:
        cal.close()
    budget = 120.0 / max(1, args.steps + args.warmup)
    S = int(max(1, min(T, budget / max(per_tok, 1e-12))))
    so = ShardedOracle(token_prefix(w, S), cores)
    try:
        bd, bc = algorithmic_bytes(S, H, K, E, P, so.R, fp8)
        for _ in range(args.warmup):
            so.one_pass()
        times = [sum(so.one_pass()) for _ in range(args.steps)]
    finally:
        so.close()
    ms = statistics.mean(times) * 1e3
    value = (bd + bc) / (ms * 1e-3) / 1e9
    sample = (f"{'all' if S == T else 'the first'} {S} of {T} tokens of the {args.workload} "
              f"workload per step: layout serial, {'FP8' if fp8 else 'BF16'} dispatch and "
              f"combine over {len(so.shards)} token shards in {so.threads} threads (C oracle)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE_TEXT[fp8],
        "data": "synthetic",
        "config": workload_config(args.workload, w, R_full, bd_full + bc_full, args.seed, world),
        "sample_tokens": S,
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": so.threads,
                         "host_cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--extra-steps", type=int, default=50)
    ap.add_argument("--eager", action="store_true", help="launch eagerly instead of CUDA graphs")
    ap.add_argument("--l2-flush", choices=("none", "write", "read"), default="none")
    ap.add_argument("--steps-per-graph", type=int, default=10,
                    help="whole steps captured in one CUDA graph for the headline timing")
    ap.add_argument("--workload", choices=("normal", "skew", "bf16", "stress"), default="normal",
                    help="workload of the timed step (the headline metric is quoted on normal)")
    ap.add_argument("--no-extra", action="store_true", help="skip the extra configs")
    ap.add_argument("--extras", default=None,
                    help="comma-separated subset of the extra configs to run (backward, dedup, "
                         "peer, epgroup, lb, ll, skew, bf16, stress); all by default")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lb-scale", type=int, default=1,
                    help="divide the redundant-expert per-slot sizes by this (small profiling case)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.steps_per_graph < 1:
        ap.error("--steps-per-graph must be at least 1")
    rank, world, _ = env_rank()
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 must be launched with torch.distributed.run (one rank per GPU)")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
