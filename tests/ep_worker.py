"""One rank of the multi-process EpGroup test (spawned by tests/test_gpu_ep.py).

Every rank draws every rank's tokens from fixed seeds, so it can compute with the
oracle both what it should receive (each source's partition-r rows of a one-GPU
dispatch with P = world) and its own combine result."""
import datetime
import os
import sys

import numpy as np


def run(rank: int, world: int, port: int, out_dir: str) -> None:
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for p in (root, os.path.join(root, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    status = "failed"
    try:
        import combine_get_dispatch_05_b200 as ep
        import oracle
        from gpu_path import bf16_to_u16, dev_u16_as_bf16, torch_identity_expert
        from workloads import make_custom

        E, H, K = 64, 256, 6
        tokens = [150 + 71 * r for r in range(world)]
        loads = [make_custom(tokens[r], H, K, E, world, seed=100 + r, mask_frac=0.1)
                 for r in range(world)]
        w = loads[rank]
        g = ep.EpGroup(E)
        x = dev_u16_as_bf16(w.x)
        idx = torch.from_numpy(w.topk_idx).cuda()
        wts = torch.from_numpy(w.topk_weights).cuda()
        (rq, rs), ri, rw, per_expert, ctx = g.dispatch(x, idx, wts)

        # received rows: each source's partition-`rank` slice, sources in rank order
        epp = E // world
        want_q, want_s, want_i, want_w, want_cnt = [], [], [], [], []
        for s, ws in enumerate(loads):
            d = oracle.dispatch(ws.x, ws.topk_idx, ws.topk_weights, E, world)
            lo, hi = d["expert_offset"][rank * epp], d["expert_offset"][(rank + 1) * epp]
            want_q.append(d["recv_x"][lo:hi])
            want_s.append(d["recv_scales"][lo:hi])
            want_i.append(d["recv_topk_idx"][lo:hi])
            want_w.append(d["recv_topk_weights"][lo:hi])
            want_cnt.append(d["num_tokens_per_expert"][rank * epp:(rank + 1) * epp])
        assert np.array_equal(rq.view(torch.uint8).cpu().numpy(), np.concatenate(want_q))
        assert np.array_equal(rs.cpu().numpy().view(np.uint32),
                              np.concatenate(want_s).view(np.uint32))
        assert np.array_equal(ri.cpu().numpy(), np.concatenate(want_i))
        assert np.array_equal(rw.cpu().numpy().view(np.uint32),
                              np.concatenate(want_w).view(np.uint32))
        assert np.array_equal(per_expert.cpu().numpy(), np.stack(want_cnt))

        # identity experts on the received rows, then combine back at the source
        y = g.combine(torch_identity_expert(rq.view(torch.uint8), rs), ctx, wts)
        mine = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, E, world)
        eo = oracle.identity_expert(mine["recv_x"], mine["recv_scales"])
        y_ref, st = oracle.combine(eo, mine["row_of"], w.topk_weights)
        assert st == 0
        assert np.array_equal(bf16_to_u16(y), y_ref)

        # BF16 payload: rows copied bit for bit, and back
        recv_b, ri_b, rw_b, per_b, ctx_b = g.dispatch(x, idx, wts, use_fp8=False)
        want_b = []
        for ws in loads:
            d = oracle.dispatch(ws.x, ws.topk_idx, ws.topk_weights, E, world, quant="none")
            lo, hi = d["expert_offset"][rank * epp], d["expert_offset"][(rank + 1) * epp]
            want_b.append(d["recv_x"][lo:hi])
        assert np.array_equal(bf16_to_u16(recv_b), np.concatenate(want_b))
        y_b = g.combine(recv_b, ctx_b, wts)
        mine_b = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, E, world, quant="none")
        y_ref_b, _ = oracle.combine(mine_b["recv_x"], mine_b["row_of"], w.topk_weights)
        assert np.array_equal(bf16_to_u16(y_b), y_ref_b)
        assert ep.ep_read_status(g.workspace) == 0
        status = "ok"
    finally:
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(status)
        dist.destroy_process_group()


def run_peer(rank: int, world: int, port: int, out_dir: str) -> None:
    """EpGroup(transport="peer") with every kernel real.  With one rank the region the
    rank allocates (ep_ipc_alloc) is the only one, so no peer mapping is opened: this
    runs the allocation, the views over it, the tables, layout, count gather, plan,
    peer dispatch, barriers, peer combine and close() on the GPU."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for p in (root, os.path.join(root, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    status = "failed"
    g = None
    try:
        import combine_get_dispatch_05_b200 as ep
        import oracle
        from gpu_path import bf16_to_u16, dev_u16_as_bf16
        from workloads import make_custom

        E, H, K = 32, 512, 4
        w = make_custom(333, H, K, E, world, seed=120 + rank, mask_frac=0.1)
        g = ep.EpGroup(E, transport="peer", hidden=H, max_tokens=512, ll_max_tokens=384)
        x = dev_u16_as_bf16(w.x)
        idx = torch.from_numpy(w.topk_idx).cuda()
        wts = torch.from_numpy(w.topk_weights).cuda()
        for quant in ("fp8", "none", "fp8"):  # the region is reused across steps
            recv_x, ri, rw, per_expert, ctx = g.dispatch(x, idx, wts, use_fp8=quant == "fp8")
            d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, E, world, quant=quant)
            R = int(d["num_recv"][0])
            assert ctx.recv_rows == R
            if quant == "fp8":
                assert np.array_equal(recv_x[0].view(torch.uint8).cpu().numpy(), d["recv_x"])
                assert np.array_equal(recv_x[1].cpu().numpy().view(np.uint32),
                                      d["recv_scales"].view(np.uint32))
            else:
                assert np.array_equal(bf16_to_u16(recv_x), d["recv_x"])
            assert np.array_equal(ri.cpu().numpy(), d["recv_topk_idx"])
            assert np.array_equal(rw.cpu().numpy().view(np.uint32),
                                  d["recv_topk_weights"].view(np.uint32))
            assert np.array_equal(per_expert.cpu().numpy().reshape(-1),
                                  d["num_tokens_per_expert"])
            eo = oracle.identity_expert(d["recv_x"], d["recv_scales"], quant=quant)
            out = g.expert_out_buffer(ctx)
            out.copy_(dev_u16_as_bf16(eo))
            y = g.combine(out, ctx, wts)
            y_ref, _ = oracle.combine(eo, d["row_of"], w.topk_weights)
            assert np.array_equal(bf16_to_u16(y), y_ref), quant
        # sync_sizes=False: the whole step without a host wait; then a receiver over
        # capacity, reported by the kernels instead of raised on the host
        recv_x, ri, rw, per_expert, ctx = g.dispatch(x, idx, wts, sync_sizes=False)
        d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, E, world, quant="fp8")
        R = int(d["num_recv"][0])
        assert int(ctx.recv_rows_device.item()) == R and ri.shape[0] == g._peer["capacity"]
        assert np.array_equal(recv_x[0][:R].view(torch.uint8).cpu().numpy(), d["recv_x"])
        assert np.array_equal(ri[:R].cpu().numpy(), d["recv_topk_idx"])
        eo = oracle.identity_expert(d["recv_x"], d["recv_scales"])
        out = g.expert_out_buffer(ctx)
        out[:R].copy_(dev_u16_as_bf16(eo))
        y = g.combine(out, ctx, wts)
        y_ref, _ = oracle.combine(eo, d["row_of"], w.topk_weights)
        assert np.array_equal(bf16_to_u16(y), y_ref), "no-sync"
        assert ep.ep_read_status(g.workspace) == 0
        small = ep.EpGroup(E, transport="peer", hidden=H, max_tokens=512, capacity=64)
        try:
            small.dispatch(x, idx, wts, sync_sizes=False)  # 1k+ rows for 64 slots: dropped
            assert ep.ep_read_status(small.workspace) == ep.EP_DEV_CAPACITY
        finally:
            small.close()
        for quant in ("fp8", "none"):  # one row per (token, rank), [K] expert lists
            recv_x, ri, rw, per_source, ctx = g.dispatch(x, idx, wts, use_fp8=quant == "fp8",
                                                         dedup=True)
            d = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, E, world, quant=quant)
            R = int(d["num_rows"][0])
            assert ctx.recv_rows == R and per_source.reshape(-1).tolist() == [R]
            if quant == "fp8":
                assert np.array_equal(recv_x[0].view(torch.uint8).cpu().numpy(), d["recv_x"])
                assert np.array_equal(recv_x[1].cpu().numpy().view(np.uint32),
                                      d["recv_scales"].view(np.uint32))
            else:
                assert np.array_equal(bf16_to_u16(recv_x), d["recv_x"])
            assert np.array_equal(ri.cpu().numpy(), d["recv_topk_idx"])
            assert np.array_equal(rw.cpu().numpy().view(np.uint32),
                                  d["recv_topk_weights"].view(np.uint32))
            po = oracle.partition_identity(d["recv_x"], d["recv_scales"], d["recv_topk_idx"],
                                           d["recv_topk_weights"], quant=quant)
            out = g.expert_out_buffer(ctx)
            out.copy_(dev_u16_as_bf16(po))
            y = g.combine(out, ctx, wts)
            y_ref, _ = oracle.combine_dedup(po, d["prow_of"])
            assert np.array_equal(bf16_to_u16(y), y_ref), "dedup " + quant
        for _ in range(2):  # low-latency rows (padded per-expert blocks)
            (q, s), count, ctx = g.low_latency_dispatch(x, idx)
            o = oracle.ll_dispatch(w.x, w.topk_idx, E, 384)
            assert np.array_equal(count.cpu().numpy().reshape(-1), o["recv_expert_count"])
            gq, gs = q.view(torch.uint8).cpu().numpy(), s.cpu().numpy()
            for e in range(E):
                n = int(o["recv_expert_count"][e])
                assert np.array_equal(gq[e, :n], o["recv_x"][e, :n]), e
                assert np.array_equal(gs[e, :n].view(np.uint32),
                                      o["recv_scales"][e, :n].view(np.uint32)), e
            eo = oracle.identity_expert(o["recv_x"].reshape(E * 384, H),
                                        o["recv_scales"].reshape(E * 384, H // 128))
            buf = g.ll_expert_out_buffer()
            buf.copy_(dev_u16_as_bf16(eo).view(E, 384, H))
            y = g.low_latency_combine(buf, ctx, wts)
            y_ref, _ = oracle.ll_combine(eo.reshape(E, 384, H), o["ll_row_of"], w.topk_weights)
            assert np.array_equal(bf16_to_u16(y), y_ref), "ll"
        assert ep.ep_read_status(g.workspace) == 0
        status = "ok"
    finally:
        try:
            if g is not None:
                g.close()
        finally:
            with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
                f.write(status)
            dist.destroy_process_group()


def run_peer_multi(rank: int, world: int, port: int, out_dir: str) -> None:
    """One process per GPU, NCCL: EpGroup(transport="peer") across real GPUs (IPC
    mappings, stores and loads over NVLink).  Per-expert, deduplicated and
    low-latency rows, each checked bit for bit against the oracle's one-GPU result on
    all ranks' tokens concatenated in rank order."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for p in (root, os.path.join(root, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    os.environ["NCCL_NVLS_ENABLE"] = "0"
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(rank)
    dist.init_process_group("nccl", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", rank))
    status = "failed"
    g = None
    try:
        import combine_get_dispatch_05_b200 as ep
        import oracle
        from gpu_path import bf16_to_u16, dev_u16_as_bf16
        from workloads import make_custom

        E, H, K, cap = 8 * world, 1024, 6, 96
        epp = E // world
        tokens = [96 - 17 * (r % 3) for r in range(world)]
        loads = [make_custom(tokens[r], H, K, E, world, seed=160 + r, mask_frac=0.05)
                 for r in range(world)]
        x_all = np.concatenate([l.x for l in loads])
        idx_all = np.concatenate([l.topk_idx for l in loads])
        w_all = np.concatenate([l.topk_weights for l in loads])
        t0 = sum(tokens[:rank])
        w = loads[rank]
        g = ep.EpGroup(E, transport="peer", hidden=H, max_tokens=128, ll_max_tokens=cap)
        x = dev_u16_as_bf16(w.x)
        idx = torch.from_numpy(w.topk_idx).cuda()
        wts = torch.from_numpy(w.topk_weights).cuda()

        # per-expert rows
        (q, s), ri, rw, per_expert, ctx = g.dispatch(x, idx, wts)
        d = oracle.dispatch(x_all, idx_all, w_all, E, world)
        lo, hi = d["expert_offset"][rank * epp], d["expert_offset"][(rank + 1) * epp]
        assert np.array_equal(q.view(torch.uint8).cpu().numpy(), d["recv_x"][lo:hi])
        assert np.array_equal(s.cpu().numpy().view(np.uint32),
                              d["recv_scales"][lo:hi].view(np.uint32))
        assert np.array_equal(ri.cpu().numpy(), d["recv_topk_idx"][lo:hi])
        eo_all = oracle.identity_expert(d["recv_x"], d["recv_scales"])
        out = g.expert_out_buffer(ctx)
        out.copy_(dev_u16_as_bf16(eo_all[lo:hi]))
        y = g.combine(out, ctx, wts)
        y_all, _ = oracle.combine(eo_all, d["row_of"], w_all)
        assert np.array_equal(bf16_to_u16(y), y_all[t0:t0 + tokens[rank]])

        # deduplicated rows
        (q, s), ri, rw, per_source, ctx = g.dispatch(x, idx, wts, dedup=True)
        d = oracle.dispatch_dedup(x_all, idx_all, w_all, E, world)
        lo, hi = d["part_offset"][rank], d["part_offset"][rank + 1]
        assert np.array_equal(q.view(torch.uint8).cpu().numpy(), d["recv_x"][lo:hi])
        assert np.array_equal(ri.cpu().numpy(), d["recv_topk_idx"][lo:hi])
        po_all = oracle.partition_identity(d["recv_x"], d["recv_scales"], d["recv_topk_idx"],
                                           d["recv_topk_weights"])
        out = g.expert_out_buffer(ctx)
        out.copy_(dev_u16_as_bf16(po_all[lo:hi]))
        y = g.combine(out, ctx, wts)
        y_all, _ = oracle.combine_dedup(po_all, d["prow_of"])
        assert np.array_equal(bf16_to_u16(y), y_all[t0:t0 + tokens[rank]])

        # low-latency rows
        (q, s), count, ctx = g.low_latency_dispatch(x, idx)
        gq, gc = q.view(torch.uint8).cpu().numpy(), count.cpu().numpy()
        buf = g.ll_expert_out_buffer()
        for src, l in enumerate(loads):
            o = oracle.ll_dispatch(l.x, l.topk_idx, E, cap)
            for el in range(epp):
                e = rank * epp + el
                n = int(o["recv_expert_count"][e])
                assert gc[el, src] == n
                assert np.array_equal(gq[el, src * cap:src * cap + n], o["recv_x"][e, :n])
            eo = oracle.identity_expert(o["recv_x"].reshape(E * cap, H),
                                        o["recv_scales"].reshape(E * cap, H // 128))
            eo = eo.reshape(E, cap, H)
            buf[:, src * cap:(src + 1) * cap].copy_(
                dev_u16_as_bf16(eo[rank * epp:(rank + 1) * epp].reshape(-1, H)).view(epp, cap, H))
            if src == rank:
                y_ref, _ = oracle.ll_combine(eo, o["ll_row_of"], w.topk_weights)
        y = g.low_latency_combine(buf, ctx, wts)
        assert np.array_equal(bf16_to_u16(y), y_ref)
        assert ep.ep_read_status(g.workspace) == 0
        status = "ok"
    finally:
        try:
            if g is not None:
                g.close()
        finally:
            with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
                f.write(status)
            dist.destroy_process_group()
