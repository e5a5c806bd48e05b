"""One rank of the CPU test of EpGroup's exchange (spawned by tests/test_ep_cpu.py).

The one-GPU kernels are replaced by CPU stand-ins built from the oracle, so that
what runs is the exchange itself: row counts, all_to_all splits, per-expert
counts and the return path, over gloo between real processes."""
import datetime
import os
import sys

import numpy as np


def _stand_ins(oracle, torch):
    def dispatch(x, idx, w, E, P, quant, q, s, ri, rw, lay, ws, stream=None):
        xs = x.view(torch.int16).numpy().view(np.uint16)
        d = oracle.dispatch(xs, idx.numpy(), w.numpy(), E, P, quant="fp8" if quant else "none")
        R = int(d["num_recv"][0])
        if quant:
            q[:R] = torch.from_numpy(d["recv_x"])
            s[:R] = torch.from_numpy(d["recv_scales"])
        else:
            q[:R] = torch.from_numpy(d["recv_x"].view(np.int16)).view(torch.bfloat16)
        ri[:R] = torch.from_numpy(d["recv_topk_idx"])
        rw[:R] = torch.from_numpy(d["recv_topk_weights"])
        for name in ("num_tokens_per_expert", "num_tokens_per_partition",
                     "is_token_in_partition", "expert_offset", "row_of", "num_recv"):
            getattr(lay, name).copy_(torch.from_numpy(np.ascontiguousarray(d[name])).view(
                getattr(lay, name).shape))
        lay.src_of[:R] = torch.from_numpy(d["src_of"])

    def combine(eo, lay, w, y, ws, stream=None):
        bits = eo.view(torch.int16).numpy().view(np.uint16)
        yb, _ = oracle.combine(bits, lay.row_of.numpy(), w.numpy())
        y.copy_(torch.from_numpy(yb.view(np.int16)).view(torch.bfloat16))

    return dispatch, combine


def run(rank: int, world: int, port: int, out_dir: str) -> None:
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for p in (root, os.path.join(root, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    status = "failed"
    try:
        import oracle
        from combine_get_dispatch_05_b200 import ep_group
        from workloads import make_custom

        stand_dispatch, stand_combine = _stand_ins(oracle, torch)
        ep_group._lib.ep_dispatch = stand_dispatch
        ep_group._lib.ep_combine = stand_combine
        ep_group._lib.ep_workspace_init = lambda ws, stream=None: None

        E, H, K = 48, 256, 5
        tokens = [0 if r == world - 1 and world > 2 else 90 + 37 * r for r in range(world)]
        loads = [make_custom(tokens[r], H, K, E, world, seed=200 + r, mask_frac=0.1)
                 for r in range(world)]
        w = loads[rank]
        g = ep_group.EpGroup(E, device="cpu")
        x = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16)
        idx = torch.from_numpy(w.topk_idx)
        wts = torch.from_numpy(w.topk_weights)
        epp = E // world
        for quant in ("fp8", "none"):
            recv_x, ri, rw, per_expert, ctx = g.dispatch(x, idx, wts, use_fp8=quant == "fp8")
            want_x, want_i, want_w, want_cnt = [], [], [], []
            for ws in loads:
                d = oracle.dispatch(ws.x, ws.topk_idx, ws.topk_weights, E, world, quant=quant)
                lo, hi = d["expert_offset"][rank * epp], d["expert_offset"][(rank + 1) * epp]
                want_x.append(d["recv_x"][lo:hi])
                want_i.append(d["recv_topk_idx"][lo:hi])
                want_w.append(d["recv_topk_weights"][lo:hi])
                want_cnt.append(d["num_tokens_per_expert"][rank * epp:(rank + 1) * epp])
            # identity experts: the received rows, dequantised as the oracle does
            if quant == "fp8":
                got_x = recv_x[0].view(torch.uint8).numpy()
                eo_bits = oracle.identity_expert(got_x, recv_x[1].numpy())
            else:
                got_x = recv_x.view(torch.int16).numpy().view(np.uint16)
                eo_bits = oracle.identity_expert(got_x, None, quant="none")
            assert np.array_equal(got_x, np.concatenate(want_x)), quant
            assert np.array_equal(ri.numpy(), np.concatenate(want_i)), quant
            assert np.array_equal(rw.numpy().view(np.uint32),
                                  np.concatenate(want_w).view(np.uint32)), quant
            assert np.array_equal(per_expert.numpy(), np.stack(want_cnt)), quant
            eo = torch.from_numpy(np.ascontiguousarray(eo_bits).view(np.int16)).view(torch.bfloat16)
            y = g.combine(eo, ctx, wts)
            mine = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, E, world, quant=quant)
            eo_mine = oracle.identity_expert(mine["recv_x"], mine.get("recv_scales"), quant=quant)
            y_ref, _ = oracle.combine(eo_mine, mine["row_of"], w.topk_weights)
            assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16), y_ref), quant
        status = "ok"
    finally:
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(status)
        dist.destroy_process_group()


# ------------------------------------------------------------ peer transport --

def _peer_stand_ins(oracle, torch):
    """CPU stand-ins for the peer transport: IPC regions are POSIX shared memory
    (the handle is its name), pointer tables hold host addresses, and the plan,
    dispatch and combine move bytes through those addresses."""
    import ctypes
    from multiprocessing import resource_tracker, shared_memory

    regions = {}

    def addr(shm):
        obj = ctypes.c_char.from_buffer(shm.buf)
        a = ctypes.addressof(obj)
        del obj
        return a

    def ipc_alloc(n):
        shm = shared_memory.SharedMemory(create=True, size=n)
        a = addr(shm)
        regions[a] = shm
        return a, shm.name.encode().ljust(64, b"\0")

    def ipc_open(h):
        shm = shared_memory.SharedMemory(name=h.rstrip(b"\0").decode())
        resource_tracker.unregister(shm._name, "shared_memory")  # the owner unlinks it
        a = addr(shm)
        regions[a] = shm
        return a

    def ipc_close(a):
        regions.pop(a).close()

    def ipc_free(a):
        shm = regions.pop(a)
        shm.close()
        shm.unlink()

    def device_bytes(ptr, n, device):
        return torch.frombuffer((ctypes.c_uint8 * n).from_address(ptr), dtype=torch.uint8)

    def layout(idx, E, P, lay, ws, stream=None):
        d = oracle.layout(idx.numpy(), E, P)
        for name in ("num_tokens_per_expert", "num_tokens_per_partition",
                     "is_token_in_partition", "expert_offset", "row_of", "num_recv"):
            t = getattr(lay, name)
            t.copy_(torch.from_numpy(np.ascontiguousarray(d[name])).view(t.shape))
        lay.src_of[:len(d["src_of"])] = torch.from_numpy(d["src_of"])

    def plan(counts, rank, expert_offset, cap, dst, rc, ro, ws, stream=None):
        c = counts.numpy().astype(np.int64)
        W, E = c.shape
        epp = E // W
        tot, before = c.sum(0), c[:rank].sum(0)
        base = np.zeros(E, np.int64)
        for q in range(W):
            seg = tot[q * epp:(q + 1) * epp]
            base[q * epp:(q + 1) * epp] = np.concatenate([[0], np.cumsum(seg)[:-1]])
        dst.copy_(torch.from_numpy((base + before - expert_offset.numpy()[:E]).astype(np.int32)))
        mine = tot[rank * epp:(rank + 1) * epp]
        rc.copy_(torch.from_numpy(mine.astype(np.int32)))
        ro.copy_(torch.from_numpy(np.concatenate([[0], np.cumsum(mine)]).astype(np.int32)))

    def put(address, arr):
        arr = np.ascontiguousarray(arr)
        ctypes.memmove(int(address), arr.ctypes.data, arr.nbytes)

    def get(address, n):
        return np.frombuffer((ctypes.c_uint8 * n).from_address(int(address)), np.uint8).copy()

    def dispatch(x, idx, w, E, W, quant, lay, dst, tables, ws, stream=None):
        xs = x.view(torch.int16).numpy().view(np.uint16)
        ids = idx.numpy()
        K = ids.shape[1]
        d = oracle.dispatch(xs, ids, w.numpy(), E, W, quant="fp8" if quant else "none")
        epp, H = E // W, xs.shape[1]
        off = dst.numpy()
        for r, src in enumerate(d["src_of"]):
            t, k = divmod(int(src), K)
            e = int(ids[t, k])
            p, row = e // epp, r + int(off[e])
            rx = d["recv_x"][r]
            put(tables.recv_x[p] + row * rx.nbytes, rx)
            if quant:
                put(tables.recv_scales[p] + row * (H // 128) * 4, d["recv_scales"][r])
            put(tables.recv_topk_idx[p] + row * 4, d["recv_topk_idx"][r:r + 1])
            put(tables.recv_topk_weights[p] + row * 4, d["recv_topk_weights"][r:r + 1])

    def combine(tables, lay, idx, dst, w, y, E, W, ws, stream=None):
        ids, ro = idx.numpy(), lay.row_of.numpy()
        T, K = ids.shape
        H = y.shape[1]
        epp, off = E // W, dst.numpy()
        rows = np.zeros((max(T * K, 1), H), np.uint16)
        row_of = np.full((T, K), -1, np.int32)
        for t in range(T):
            for k in range(K):
                if ro[t, k] >= 0:
                    e = int(ids[t, k])
                    a = tables.expert_out[e // epp] + (int(ro[t, k]) + int(off[e])) * H * 2
                    rows[t * K + k] = get(a, H * 2).view(np.uint16)
                    row_of[t, k] = t * K + k
        yb, _ = oracle.combine(rows, row_of, w.numpy())
        y.copy_(torch.from_numpy(yb.view(np.int16)).view(torch.bfloat16))

    def layout_dedup(idx, E, P, lay, ws, stream=None):
        ids = idx.numpy()
        d = oracle.dispatch_dedup(np.zeros((ids.shape[0], 128), np.uint16), ids,
                                  np.zeros(ids.shape, np.float32), E, P, quant="none")
        lay.num_tokens_per_expert.copy_(torch.from_numpy(d["part_count"]))
        lay.num_tokens_per_partition.copy_(torch.from_numpy(d["part_count"]))
        lay.expert_offset.copy_(torch.from_numpy(d["part_offset"]))
        lay.row_of.copy_(torch.from_numpy(d["prow_of"]))
        lay.is_token_in_partition.copy_(torch.from_numpy((d["prow_of"] >= 0).astype(np.uint8)))
        lay.src_of[:len(d["src_tok"])] = torch.from_numpy(d["src_tok"])
        lay.num_recv.fill_(int(d["num_rows"][0]))

    def dispatch_dedup(x, idx, w, E, W, quant, lay, dst, tables, ws, stream=None):
        xs = x.view(torch.int16).numpy().view(np.uint16)
        H = xs.shape[1]
        d = oracle.dispatch_dedup(xs, idx.numpy(), w.numpy(), E, W, quant="fp8" if quant else "none")
        off, po = dst.numpy(), d["part_offset"]
        for q in range(W):
            for r in range(int(po[q]), int(po[q + 1])):
                row = r + int(off[q])
                rx = d["recv_x"][r]
                put(tables.recv_x[q] + row * rx.nbytes, rx)
                if quant:
                    put(tables.recv_scales[q] + row * (H // 128) * 4, d["recv_scales"][r])
                put(tables.recv_topk_idx[q] + row * d["recv_topk_idx"][r].nbytes,
                    d["recv_topk_idx"][r])
                put(tables.recv_topk_weights[q] + row * d["recv_topk_weights"][r].nbytes,
                    d["recv_topk_weights"][r])

    def combine_dedup(tables, lay, dst, y, W, ws, stream=None):
        pr, off = lay.row_of.numpy(), dst.numpy()
        T, H = y.shape
        rows = np.zeros((max(T * W, 1), H), np.uint16)
        prow = np.full((T, W), -1, np.int32)
        for t in range(T):
            for q in range(W):
                if pr[t, q] >= 0:
                    a = tables.expert_out[q] + (int(pr[t, q]) + int(off[q])) * H * 2
                    rows[t * W + q] = get(a, H * 2).view(np.uint16)
                    prow[t, q] = t * W + q
        yb, _ = oracle.combine_dedup(rows, prow)
        y.copy_(torch.from_numpy(yb.view(np.int16)).view(torch.bfloat16))

    def ll_dispatch(x, idx, cap, E, W, rank, tx, ts, tc, h, ws, stream=None):
        xs = x.view(torch.int16).numpy().view(np.uint16)
        H = xs.shape[1]
        o = oracle.ll_dispatch(xs, idx.numpy(), E, cap)
        epp = E // W
        for e in range(E):
            q, el, n = e // epp, e % epp, int(o["recv_expert_count"][e])
            put(tc[q] + (el * W + rank) * 4, np.array([n], np.int32))
            for j in range(n):
                row = (el * W + rank) * cap + j
                put(tx[q] + row * H, o["recv_x"][e, j])
                put(ts[q] + row * (H // 128) * 4, o["recv_scales"][e, j])
        h.row_of.copy_(torch.from_numpy(o["ll_row_of"]))
        h.src_of.copy_(torch.from_numpy(o["ll_src_of"]))

    def ll_combine(te, idx, h, w, y, E, W, rank, ws, stream=None):
        ids, ro = idx.numpy(), h.row_of.numpy()
        T, K = ids.shape
        H, cap, epp = y.shape[1], h.num_max_tokens, E // W
        rows = np.zeros((max(T * K, 1), H), np.uint16)
        row_of = np.full((T, K), -1, np.int32)
        for t in range(T):
            for k in range(K):
                if ro[t, k] >= 0:
                    e = int(ids[t, k])
                    j = int(ro[t, k]) - e * cap
                    a = te[e // epp] + (((e % epp) * W + rank) * cap + j) * H * 2
                    rows[t * K + k] = get(a, H * 2).view(np.uint16)
                    row_of[t, k] = t * K + k
        yb, _ = oracle.combine(rows, row_of, w.numpy())
        y.copy_(torch.from_numpy(yb.view(np.int16)).view(torch.bfloat16))

    return dict(ep_ipc_alloc=ipc_alloc, ep_ipc_open=ipc_open, ep_ipc_close=ipc_close,
                ep_peer_low_latency_dispatch=ll_dispatch, ep_peer_low_latency_combine=ll_combine,
                ep_ipc_free=ipc_free, device_bytes=device_bytes, ep_get_dispatch_layout=layout,
                ep_peer_plan=plan, ep_peer_dispatch=dispatch, ep_peer_combine=combine,
                ep_get_dispatch_layout_dedup=layout_dedup, ep_peer_dispatch_dedup=dispatch_dedup,
                ep_peer_combine_dedup=combine_dedup,
                ep_workspace_init=lambda ws, stream=None: None)


def run_peer(rank: int, world: int, port: int, out_dir: str) -> None:
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for p in (root, os.path.join(root, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    status = "failed"
    g = None
    try:
        import oracle
        from combine_get_dispatch_05_b200 import ep_group
        from workloads import make_custom

        for name, fn in _peer_stand_ins(oracle, torch).items():
            setattr(ep_group._lib, name, fn)

        E, H, K = 24, 256, 4
        epp = E // world
        tokens = [0 if r == world - 1 and world > 2 else 70 + 29 * r for r in range(world)]
        loads = [make_custom(tokens[r], H, K, E, world, seed=300 + r, mask_frac=0.1)
                 for r in range(world)]
        x_all = np.concatenate([w.x for w in loads])
        idx_all = np.concatenate([w.topk_idx for w in loads])
        w_all = np.concatenate([w.topk_weights for w in loads])
        t0 = sum(tokens[:rank])
        w = loads[rank]
        cap = 128
        g = ep_group.EpGroup(E, device="cpu", transport="peer", hidden=H, max_tokens=128,
                             ll_max_tokens=cap)
        x = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16)
        idx = torch.from_numpy(w.topk_idx)
        wts = torch.from_numpy(w.topk_weights)
        for step, quant in enumerate(("fp8", "none", "fp8")):  # the buffers are reused
            if step == 2:  # through the receive hook: the oracle runs while rows travel
                recv_x, ri, rw, per_expert, ctx, hook = g.dispatch(
                    x, idx, wts, use_fp8=quant == "fp8", return_recv_hook=True)
                d = oracle.dispatch(x_all, idx_all, w_all, E, world, quant=quant)
                hook()
                hook()  # a second call is a no-op
            else:
                recv_x, ri, rw, per_expert, ctx = g.dispatch(x, idx, wts, use_fp8=quant == "fp8")
                d = oracle.dispatch(x_all, idx_all, w_all, E, world, quant=quant)
            lo, hi = d["expert_offset"][rank * epp], d["expert_offset"][(rank + 1) * epp]
            if quant == "fp8":
                got = recv_x[0].view(torch.uint8).numpy()
                assert np.array_equal(recv_x[1].numpy().view(np.uint32),
                                      d["recv_scales"][lo:hi].view(np.uint32))
            else:
                got = recv_x.view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(got, d["recv_x"][lo:hi]), quant
            assert np.array_equal(ri.numpy(), d["recv_topk_idx"][lo:hi]), quant
            assert np.array_equal(rw.numpy().view(np.uint32),
                                  d["recv_topk_weights"][lo:hi].view(np.uint32)), quant
            want_cnt = np.stack([oracle.layout(l.topk_idx, E, world)["num_tokens_per_expert"]
                                 [rank * epp:(rank + 1) * epp] for l in loads])
            assert np.array_equal(per_expert.numpy(), want_cnt), quant
            assert ctx.recv_counts == want_cnt.sum(1).tolist()
            eo_all = oracle.identity_expert(d["recv_x"], d["recv_scales"], quant=quant)
            buf = g.expert_out_buffer(ctx)
            buf.copy_(torch.from_numpy(eo_all[lo:hi].view(np.int16)).view(torch.bfloat16))
            y = g.combine(buf, ctx, wts)
            y_all, _ = oracle.combine(eo_all, d["row_of"], w_all)
            assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16),
                                  y_all[t0:t0 + tokens[rank]]), quant
        # sync_sizes=False: nothing waits on the host; capacity-sized views whose first
        # recv_rows_device rows are this step's, counts read on request
        for dedup in (False, True):
            recv_x, ri, rw, per, ctx = g.dispatch(x, idx, wts, dedup=dedup, sync_sizes=False)
            assert not ctx.sizes_synced and ri.shape[0] == g._peer["capacity"]
            if dedup:
                d = oracle.dispatch_dedup(x_all, idx_all, w_all, E, world, quant="fp8")
                lo, hi = d["part_offset"][rank], d["part_offset"][rank + 1]
            else:
                d = oracle.dispatch(x_all, idx_all, w_all, E, world, quant="fp8")
                lo, hi = d["expert_offset"][rank * epp], d["expert_offset"][(rank + 1) * epp]
            n = int(ctx.recv_rows_device.item())
            assert n == hi - lo and ctx.recv_rows == n
            assert np.array_equal(recv_x[0][:n].view(torch.uint8).numpy(), d["recv_x"][lo:hi])
            assert np.array_equal(ri[:n].numpy(), d["recv_topk_idx"][lo:hi])
            assert sum(ctx.recv_counts) == n and len(ctx.send_counts) == world
            buf = g.expert_out_buffer(ctx)
            assert buf.shape[0] == g._peer["capacity"]
            if dedup:
                po_all = oracle.partition_identity(d["recv_x"], d["recv_scales"],
                                                   d["recv_topk_idx"], d["recv_topk_weights"])
                buf[:n].copy_(torch.from_numpy(po_all[lo:hi].view(np.int16)).view(torch.bfloat16))
                y_all, _ = oracle.combine_dedup(po_all, d["prow_of"])
            else:
                eo_all = oracle.identity_expert(d["recv_x"], d["recv_scales"])
                buf[:n].copy_(torch.from_numpy(eo_all[lo:hi].view(np.int16)).view(torch.bfloat16))
                y_all, _ = oracle.combine(eo_all, d["row_of"], w_all)
            y = g.combine(buf, ctx, wts)
            assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16),
                                  y_all[t0:t0 + tokens[rank]]), f"no-sync dedup={dedup}"
            # the buffers' views are kept between calls: reshaping a returned tensor in
            # place must not change what the next call returns
            shapes = (tuple(recv_x[0].shape), tuple(ri.shape), tuple(buf.shape))
            recv_x[0].unsqueeze_(0)
            ri.unsqueeze_(0)
            buf.unsqueeze_(0)
            again = g.dispatch(x, idx, wts, dedup=dedup, sync_sizes=False)
            assert (tuple(again[0][0].shape), tuple(again[1].shape),
                    tuple(g.expert_out_buffer(again[4]).shape)) == shapes
            g.combine(g.expert_out_buffer(again[4]), again[4], wts)
        for quant in ("fp8", "none"):  # one row per (token, rank)
            recv_x, ri, rw, per_source, ctx = g.dispatch(x, idx, wts, use_fp8=quant == "fp8",
                                                         dedup=True)
            d = oracle.dispatch_dedup(x_all, idx_all, w_all, E, world, quant=quant)
            lo, hi = d["part_offset"][rank], d["part_offset"][rank + 1]
            if quant == "fp8":
                got = recv_x[0].view(torch.uint8).numpy()
                assert np.array_equal(recv_x[1].numpy().view(np.uint32),
                                      d["recv_scales"][lo:hi].view(np.uint32))
            else:
                got = recv_x.view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(got, d["recv_x"][lo:hi]), quant
            assert np.array_equal(ri.numpy(), d["recv_topk_idx"][lo:hi]), quant
            assert np.array_equal(rw.numpy().view(np.uint32),
                                  d["recv_topk_weights"][lo:hi].view(np.uint32)), quant
            want = [int(oracle.dispatch_dedup(l.x, l.topk_idx, l.topk_weights, E, world,
                                              quant=quant)["part_count"][rank]) for l in loads]
            assert per_source.reshape(-1).tolist() == want and ctx.recv_counts == want
            po_all = oracle.partition_identity(d["recv_x"], d["recv_scales"], d["recv_topk_idx"],
                                               d["recv_topk_weights"], quant=quant)
            buf = g.expert_out_buffer(ctx)
            buf.copy_(torch.from_numpy(po_all[lo:hi].view(np.int16)).view(torch.bfloat16))
            y = g.combine(buf, ctx, wts)
            y_all, _ = oracle.combine_dedup(po_all, d["prow_of"])
            assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16),
                                  y_all[t0:t0 + tokens[rank]]), "dedup " + quant
        for step in range(2):  # low-latency rows: padded per-expert blocks, one per source
            if step == 0:
                (q, s), count, ctx, hook = g.low_latency_dispatch(x, idx, return_recv_hook=True)
                hook()
            else:
                (q, s), count, ctx = g.low_latency_dispatch(x, idx)
            got_q, got_s, got_c = q.view(torch.uint8).numpy(), s.numpy(), count.numpy()
            for src, l in enumerate(loads):
                o = oracle.ll_dispatch(l.x, l.topk_idx, E, cap)
                for el in range(epp):
                    e = rank * epp + el
                    n = int(o["recv_expert_count"][e])
                    assert got_c[el, src] == n
                    blk = slice(src * cap, src * cap + n)
                    assert np.array_equal(got_q[el, blk], o["recv_x"][e, :n])
                    assert np.array_equal(got_s[el, blk].view(np.uint32),
                                          o["recv_scales"][e, :n].view(np.uint32))
                eo = oracle.identity_expert(o["recv_x"].reshape(E * cap, H),
                                            o["recv_scales"].reshape(E * cap, H // 128))
                eo = eo.reshape(E, cap, H)
                buf = g.ll_expert_out_buffer()
                buf[:, src * cap:(src + 1) * cap].copy_(torch.from_numpy(
                    eo[rank * epp:(rank + 1) * epp].view(np.int16)).view(torch.bfloat16))
                if src == rank:
                    y_ref, _ = oracle.ll_combine(eo, o["ll_row_of"], w.topk_weights)
            y = g.low_latency_combine(g.ll_expert_out_buffer(), ctx, wts)
            assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16), y_ref), "ll"

        # error paths: each raises on every rank alike, and the group stays usable
        def raises(exc, fn):
            try:
                fn()
            except exc:
                return True
            return False

        assert raises(ValueError, lambda: g.dispatch(x[:, :128].contiguous(), idx, wts))  # hidden
        recv_x, ri, rw, per_expert, ctx = g.dispatch(x, idx, wts)
        assert raises(ValueError, lambda: g.combine(torch.empty_like(g.expert_out_buffer(ctx)),
                                                    ctx, wts))
        g.combine(g.expert_out_buffer(ctx), ctx, wts)  # the step completes normally
        small = ep_group.EpGroup(E, device="cpu", transport="peer", hidden=H, max_tokens=128,
                                 capacity=8)
        try:
            assert raises(ValueError, lambda: small.dispatch(x, idx, wts))  # over capacity
            assert raises(ValueError, lambda: small.dispatch(x, idx, wts, dedup=True))
            assert raises(RuntimeError, lambda: small.low_latency_dispatch(x, idx))
        finally:
            small.close()
        (q, s), count, ctx = g.low_latency_dispatch(x, idx)  # still usable
        g.low_latency_combine(g.ll_expert_out_buffer(), ctx, wts)
        status = "ok"
    finally:
        try:
            if g is not None:
                g.close()
        finally:
            with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
                f.write(status)
            dist.destroy_process_group()
