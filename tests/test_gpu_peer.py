"""Expert parallelism across GPUs through peer memory, every rank emulated on the one
GPU: the W ranks' receive buffers are separate device allocations and the pointer
tables hold their addresses, as they would hold IPC-mapped peers'.  Each rank's
layout, plan, dispatch and combine are launched in turn on one stream; no kernel
waits on another.

Rank p's receive rows must equal, byte for byte, partition p's rows of the oracle's
one-GPU dispatch of all ranks' tokens concatenated in rank order, and each rank's
combine must equal the oracle's combine of its tokens.  Rows past what a rank
receives stay unwritten and every buffer's tail canary is intact.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
from workloads import make_custom, make_workload  # noqa: E402

from gpu_path import CANARY, Guarded, bf16_to_u16, dev_u16_as_bf16, new_workspace, quant_code  # noqa: E402


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import combine_get_dispatch_05_b200 as m
    return m


def _concat(loads):
    x = np.concatenate([w.x for w in loads])
    idx = np.concatenate([w.topk_idx for w in loads])
    wts = np.concatenate([w.topk_weights for w in loads])
    return x, idx, wts


def _run(ep, loads, E, W, quant, capacity):
    H = loads[0].hidden
    fp8 = quant != "none"
    cap = capacity
    bufs = []
    for _ in range(W):
        bufs.append(dict(
            x=Guarded((cap, H), torch.uint8 if fp8 else torch.bfloat16),
            s=Guarded((cap, H // 128), torch.float32) if fp8 else None,
            i=Guarded((cap,), torch.int32), w=Guarded((cap,), torch.float32),
            eo=Guarded((cap, H), torch.bfloat16)))
    tables = ep.PeerTables.from_addresses(
        "cuda", cap, [b["x"].t.data_ptr() for b in bufs],
        [b["s"].t.data_ptr() if fp8 else 0 for b in bufs],
        [b["i"].t.data_ptr() for b in bufs], [b["w"].t.data_ptr() for b in bufs],
        [b["eo"].t.data_ptr() for b in bufs])
    ranks = []
    for w in loads:
        T, K = w.num_tokens, w.num_topk
        r = dict(x=dev_u16_as_bf16(w.x), idx=torch.from_numpy(w.topk_idx).cuda(),
                 wts=torch.from_numpy(w.topk_weights).cuda(),
                 lay=ep.Layout.empty(T, K, E, W, "cuda"), ws=new_workspace(ep, T, E, W))
        ep.ep_get_dispatch_layout(r["idx"], E, W, r["lay"], r["ws"])
        ranks.append(r)
    counts = torch.stack([r["lay"].num_tokens_per_expert for r in ranks]).contiguous()
    epp = E // W
    for s, r in enumerate(ranks):
        r["dst"] = torch.empty(E, dtype=torch.int32, device="cuda")
        r["rc"] = torch.empty(epp, dtype=torch.int32, device="cuda")
        r["ro"] = torch.empty(epp + 1, dtype=torch.int32, device="cuda")
        ep.ep_peer_plan(counts, s, r["lay"].expert_offset, cap, r["dst"], r["rc"], r["ro"], r["ws"])
    for r in ranks:
        ep.ep_peer_dispatch(r["x"], r["idx"], r["wts"], E, W, quant_code(ep, quant), r["lay"],
                            r["dst"], tables, r["ws"])
    torch.cuda.synchronize()
    return bufs, tables, ranks


def _check(ep, loads, E, W, quant, capacity=None, drop=()):
    """drop: partitions whose receive total is expected to exceed `capacity`."""
    H = loads[0].hidden
    fp8 = quant != "none"
    epp = E // W
    x, idx, wts = _concat(loads)
    d = oracle.dispatch(x, idx, wts, E, W, quant=quant)
    off = d["expert_offset"]
    part_rows = [int(off[(p + 1) * epp] - off[p * epp]) for p in range(W)]
    cap = capacity if capacity is not None else max(max(part_rows), 1) + 3
    bufs, tables, ranks = _run(ep, loads, E, W, quant, cap)

    status = [ep.ep_read_status(r["ws"]) for r in ranks]
    if drop:
        assert all(st & ep.EP_DEV_CAPACITY for st in status), status
    else:
        assert status == [0] * W, status

    # receive buffers: partition p's slice of the concatenated dispatch
    for p in range(W):
        lo, n = int(off[p * epp]), part_rows[p]
        b = bufs[p]
        row_bytes = H * (1 if fp8 else 2)
        if p in drop:
            assert bool((b["x"].raw == CANARY).all().item()), f"rank {p} was written"
            n = 0
        else:
            if fp8:
                assert np.array_equal(b["x"].t[:n].cpu().numpy(), d["recv_x"][lo:lo + n]), p
                assert np.array_equal(b["s"].t[:n].cpu().numpy().view(np.uint32),
                                      d["recv_scales"][lo:lo + n].view(np.uint32)), p
            else:
                assert np.array_equal(bf16_to_u16(b["x"].t[:n]), d["recv_x"][lo:lo + n]), p
            assert np.array_equal(b["i"].t[:n].cpu().numpy(), d["recv_topk_idx"][lo:lo + n]), p
            assert np.array_equal(b["w"].t[:n].cpu().numpy().view(np.uint32),
                                  d["recv_topk_weights"][lo:lo + n].view(np.uint32)), p
        assert bool((b["x"].raw[n * row_bytes:] == CANARY).all().item()), p
        assert all(g.canary_ok() for g in (b["x"], b["i"], b["w"]) + ((b["s"],) if fp8 else ()))
        # the plan's receive counts and offsets for rank p
        rc, ro = ranks[p]["rc"].cpu().numpy(), ranks[p]["ro"].cpu().numpy()
        if p in drop:
            assert not rc.any() and not ro.any()
        else:
            want = d["num_tokens_per_expert"][p * epp:(p + 1) * epp]
            assert np.array_equal(rc, want)
            assert np.array_equal(ro, np.concatenate([[0], np.cumsum(want)]).astype(np.int32))

    # expert outputs: identity experts on each rank's rows, written into its buffer
    eo_all = oracle.identity_expert(d["recv_x"], d.get("recv_scales"), quant=quant)
    for p in range(W):
        lo, n = int(off[p * epp]), part_rows[p]
        if p not in drop and n:
            bufs[p]["eo"].t[:n].copy_(dev_u16_as_bf16(eo_all[lo:lo + n]))
    torch.cuda.synchronize()

    # combine on every rank, reading the owners' expert outputs
    row_of = d["row_of"].copy()
    if drop:
        part = np.where(idx >= 0, idx // epp, -1)
        row_of[np.isin(part, list(drop))] = -1
    y_all, _ = oracle.combine(eo_all, row_of, wts)
    t0 = 0
    for s, (w, r) in enumerate(zip(loads, ranks)):
        T = w.num_tokens
        y = Guarded((T, H), torch.bfloat16)
        ep.ep_peer_combine(tables, r["lay"], r["idx"], r["dst"], r["wts"], y.t, E, W, r["ws"])
        torch.cuda.synchronize()
        assert np.array_equal(bf16_to_u16(y.t), y_all[t0:t0 + T]), s
        assert y.canary_ok()
        st = ep.ep_read_status(r["ws"])
        dropped_here = drop and bool(np.isin(np.where(w.topk_idx >= 0, w.topk_idx // epp, -1),
                                             list(drop)).any())
        assert bool(st & ep.EP_DEV_INDEX_RANGE) == bool(dropped_here), (s, st)
        t0 += T


@pytest.mark.parametrize("quant", ["fp8", "fp8_pow2", "none"])
def test_peer_two_ranks_ragged(ep, quant):
    # H = 256: two scale blocks per row, 8 bytes (the per-lane scale path);
    # masked slots; different batch sizes per rank
    loads = [make_custom(T, 256, 4, 16, 2, seed=40 + s, mask_frac=0.05)
             for s, T in enumerate([300, 173])]
    _check(ep, loads, 16, 2, quant)


def test_peer_four_ranks_duplicates_and_empty_rank(ep):
    # a rank with no tokens; duplicate experts within a token (separate rows)
    loads = [make_custom(T, 1024, 8, 32, 4, seed=50 + s, duplicates=True)
             for s, T in enumerate([129, 0, 260, 64])]
    _check(ep, loads, 32, 4, "fp8")


def test_peer_three_ranks_bf16(ep):
    loads = [make_custom(T, 384, 6, 24, 3, seed=60 + s, mask_frac=0.1)
             for s, T in enumerate([200, 57, 311])]
    _check(ep, loads, 24, 3, "none")


def test_peer_eight_ranks_normal_routing(ep):
    # 8 ranks x 512 tokens of the normal workload (hidden 7168, top-8 of 256
    # experts under top-4-of-8-group routing): 4096 tokens in all
    loads = [make_workload("normal", seed=70 + s, num_tokens=512) for s in range(8)]
    _check(ep, loads, 256, 8, "fp8")


def test_peer_capacity_overflow_drops_one_rank(ep):
    # rank 0's experts take every token's first choice: its receive total exceeds
    # the capacity, so it receives nothing; rank 1 receives all of its rows
    loads = [make_custom(T, 512, 2, 8, 2, seed=80 + s, hot_expert=1) for s, T in enumerate([90, 70])]
    x, idx, wts = _concat(loads)
    d = oracle.dispatch(x, idx, wts, 8, 2, quant="fp8")
    rows0 = int(d["expert_offset"][4])
    rows1 = int(d["expert_offset"][8] - d["expert_offset"][4])
    assert rows0 > rows1
    _check(ep, loads, 8, 2, "fp8", capacity=rows1, drop=(0,))


# ------------------------------------------------------- deduplicated rows --

def _check_dedup(ep, loads, E, W, quant, capacity=None, drop=()):
    H, K = loads[0].hidden, loads[0].num_topk
    fp8 = quant != "none"
    x, idx, wts = _concat(loads)
    d = oracle.dispatch_dedup(x, idx, wts, E, W, quant=quant)
    off = d["part_offset"]
    part_rows = [int(off[q + 1] - off[q]) for q in range(W)]
    cap = capacity if capacity is not None else max(max(part_rows), 1) + 5
    bufs = [dict(x=Guarded((cap, H), torch.uint8 if fp8 else torch.bfloat16),
                 s=Guarded((cap, H // 128), torch.float32) if fp8 else None,
                 i=Guarded((cap, K), torch.int32), w=Guarded((cap, K), torch.float32),
                 eo=Guarded((cap, H), torch.bfloat16)) for _ in range(W)]
    tables = ep.PeerTables.from_addresses(
        "cuda", cap, [b["x"].t.data_ptr() for b in bufs],
        [b["s"].t.data_ptr() if fp8 else 0 for b in bufs],
        [b["i"].t.data_ptr() for b in bufs], [b["w"].t.data_ptr() for b in bufs],
        [b["eo"].t.data_ptr() for b in bufs])
    ranks = []
    for w in loads:
        T = w.num_tokens
        r = dict(x=dev_u16_as_bf16(w.x), idx=torch.from_numpy(w.topk_idx).cuda(),
                 wts=torch.from_numpy(w.topk_weights).cuda(),
                 lay=ep.Layout.empty(T, W, W, W, "cuda"), ws=new_workspace(ep, T, E, W),
                 dst=torch.empty(W, dtype=torch.int32, device="cuda"),
                 rc=torch.empty(1, dtype=torch.int32, device="cuda"),
                 ro=torch.empty(2, dtype=torch.int32, device="cuda"))
        ep.ep_get_dispatch_layout_dedup(r["idx"], E, W, r["lay"], r["ws"])
        ranks.append(r)
    counts = torch.stack([r["lay"].num_tokens_per_expert for r in ranks]).contiguous()
    for s, r in enumerate(ranks):
        ep.ep_peer_plan(counts, s, r["lay"].expert_offset, cap, r["dst"], r["rc"], r["ro"], r["ws"])
    for r in ranks:
        ep.ep_peer_dispatch_dedup(r["x"], r["idx"], r["wts"], E, W, quant_code(ep, quant),
                                  r["lay"], r["dst"], tables, r["ws"])
    torch.cuda.synchronize()
    status = [ep.ep_read_status(r["ws"]) for r in ranks]
    if drop:
        assert all(st & ep.EP_DEV_CAPACITY for st in status), status
    else:
        assert status == [0] * W, status

    row_bytes = H * (1 if fp8 else 2)
    for q in range(W):
        lo, n = int(off[q]), part_rows[q]
        b = bufs[q]
        if q in drop:
            assert bool((b["x"].raw == CANARY).all().item()), f"rank {q} was written"
            n = 0
        else:
            if fp8:
                assert np.array_equal(b["x"].t[:n].cpu().numpy(), d["recv_x"][lo:lo + n]), q
                assert np.array_equal(b["s"].t[:n].cpu().numpy().view(np.uint32),
                                      d["recv_scales"][lo:lo + n].view(np.uint32)), q
            else:
                assert np.array_equal(bf16_to_u16(b["x"].t[:n]), d["recv_x"][lo:lo + n]), q
            assert np.array_equal(b["i"].t[:n].cpu().numpy(), d["recv_topk_idx"][lo:lo + n]), q
            assert np.array_equal(b["w"].t[:n].cpu().numpy().view(np.uint32),
                                  d["recv_topk_weights"][lo:lo + n].view(np.uint32)), q
            assert int(ranks[q]["rc"].item()) == n
            assert ranks[q]["ro"].cpu().tolist() == [0, n]
        assert bool((b["x"].raw[n * row_bytes:] == CANARY).all().item()), q
        assert all(g.canary_ok() for g in (b["x"], b["i"], b["w"]) + ((b["s"],) if fp8 else ()))

    # partition outputs (each received row reduced over its listed experts), then combine
    po_all = oracle.partition_identity(d["recv_x"], d["recv_scales"], d["recv_topk_idx"],
                                       d["recv_topk_weights"], quant="none" if not fp8 else "fp8")
    for q in range(W):
        lo, n = int(off[q]), part_rows[q]
        if q not in drop and n:
            bufs[q]["eo"].t[:n].copy_(dev_u16_as_bf16(po_all[lo:lo + n]))
    torch.cuda.synchronize()
    prow = d["prow_of"].copy()
    for q in drop:
        prow[:, q] = -1
    y_all, _ = oracle.combine_dedup(po_all, prow)
    t0 = 0
    for s, (w, r) in enumerate(zip(loads, ranks)):
        T = w.num_tokens
        y = Guarded((T, H), torch.bfloat16)
        ep.ep_peer_combine_dedup(tables, r["lay"], r["dst"], y.t, W, r["ws"])
        torch.cuda.synchronize()
        assert np.array_equal(bf16_to_u16(y.t), y_all[t0:t0 + T]), s
        assert y.canary_ok()
        st = ep.ep_read_status(r["ws"])
        dropped_here = bool(drop) and bool((d["prow_of"][t0:t0 + T][:, list(drop)] >= 0).any())
        assert bool(st & ep.EP_DEV_INDEX_RANGE) == dropped_here, (s, st)
        t0 += T


@pytest.mark.parametrize("quant", ["fp8", "none"])
def test_peer_dedup_two_ranks_ragged(ep, quant):
    loads = [make_custom(T, 256, 6, 16, 2, seed=90 + s, mask_frac=0.05)
             for s, T in enumerate([241, 130])]
    _check_dedup(ep, loads, 16, 2, quant)


def test_peer_dedup_four_ranks_empty_rank_pow2(ep):
    loads = [make_custom(T, 512, 8, 32, 4, seed=95 + s, duplicates=True)
             for s, T in enumerate([77, 0, 190, 33])]
    _check_dedup(ep, loads, 32, 4, "fp8_pow2")


def test_peer_dedup_eight_ranks_normal_routing(ep):
    loads = [make_workload("normal", seed=110 + s, num_tokens=512) for s in range(8)]
    _check_dedup(ep, loads, 256, 8, "fp8")


def test_peer_dedup_capacity_overflow_drops_one_rank(ep):
    loads = [make_custom(T, 512, 2, 8, 2, seed=120 + s, hot_expert=1) for s, T in enumerate([90, 70])]
    x, idx, wts = _concat(loads)
    d = oracle.dispatch_dedup(x, idx, wts, 8, 2, quant="fp8")
    rows1 = int(d["part_offset"][2] - d["part_offset"][1])
    assert int(d["part_offset"][1]) > rows1
    _check_dedup(ep, loads, 8, 2, "fp8", capacity=rows1, drop=(0,))


# ------------------------------------------------------ low-latency rows --

def _check_ll(ep, loads, E, W, cap):
    """Every rank's padded receive buffer [E/W, W*cap, H]: source s's block of local
    expert el must equal, byte for byte, the oracle's one-GPU low-latency dispatch of
    s's tokens for expert q*Epp + el (unwritten slots keep the 0xA5 fill on both
    sides); the counts and the local handle likewise; then each rank's combine."""
    H, K = loads[0].hidden, loads[0].num_topk
    epp = E // W
    bufs = [dict(x=Guarded((epp, W * cap, H), torch.uint8),
                 s=Guarded((epp, W * cap, H // 128), torch.float32),
                 c=Guarded((epp, W), torch.int32),
                 eo=Guarded((epp, W * cap, H), torch.bfloat16)) for _ in range(W)]

    def table(key):
        return torch.tensor([b[key].t.data_ptr() for b in bufs], dtype=torch.int64, device="cuda")

    tx, ts, tc, te = table("x"), table("s"), table("c"), table("eo")
    ranks, want = [], []
    for s, w in enumerate(loads):
        T = w.num_tokens
        r = dict(x=dev_u16_as_bf16(w.x), idx=torch.from_numpy(w.topk_idx).cuda(),
                 wts=torch.from_numpy(w.topk_weights).cuda(),
                 h=ep.LowLatencyHandle.empty(T, K, E, cap, "cuda"), ws=new_workspace(ep, T, E, W))
        ep.ep_peer_low_latency_dispatch(r["x"], r["idx"], cap, E, W, s, tx, ts, tc, r["h"], r["ws"])
        ranks.append(r)
        want.append(oracle.ll_dispatch(w.x, w.topk_idx, E, cap, fill=CANARY))
    torch.cuda.synchronize()
    assert [ep.ep_read_status(r["ws"]) for r in ranks] == [0] * W
    for q in range(W):
        b = bufs[q]
        gx, gs, gc = b["x"].t.cpu().numpy(), b["s"].t.cpu().numpy(), b["c"].t.cpu().numpy()
        for s in range(W):
            o = want[s]
            blk = slice(s * cap, (s + 1) * cap)
            assert np.array_equal(gx[:, blk], o["recv_x"][q * epp:(q + 1) * epp]), (q, s)
            cnt = o["recv_expert_count"][q * epp:(q + 1) * epp]
            assert np.array_equal(gc[:, s], cnt), (q, s)
            for el in range(epp):
                n = int(cnt[el])
                assert np.array_equal(gs[el, s * cap:s * cap + n].view(np.uint32),
                                      o["recv_scales"][q * epp + el, :n].view(np.uint32)), (q, s, el)
        assert all(g.canary_ok() for g in (b["x"], b["s"], b["c"]))
    for s, r in enumerate(ranks):
        assert np.array_equal(r["h"].row_of.cpu().numpy(), want[s]["ll_row_of"]), s
        so = r["h"].src_of.cpu().numpy()
        for e in range(E):  # the local handle: slot j of e holds (t, k) = src_of[e, j]
            n = int(want[s]["recv_expert_count"][e])
            assert np.array_equal(so[e, :n], want[s]["ll_src_of"][e, :n]), (s, e)

    # expert outputs: identity experts on each source's rows, placed in the owners'
    # blocks; then every rank's combine reads them back
    y_refs = []
    for s, w in enumerate(loads):
        o = want[s]
        eo = oracle.identity_expert(o["recv_x"].reshape(E * cap, H),
                                    o["recv_scales"].reshape(E * cap, H // 128)).reshape(E, cap, H)
        for q in range(W):
            bufs[q]["eo"].t[:, s * cap:(s + 1) * cap].copy_(
                dev_u16_as_bf16(eo[q * epp:(q + 1) * epp].reshape(-1, H)).view(epp, cap, H))
        y_refs.append(oracle.ll_combine(eo, o["ll_row_of"], w.topk_weights)[0])
        del eo
        want[s] = None
    torch.cuda.synchronize()
    for s, (w, r) in enumerate(zip(loads, ranks)):
        y = Guarded((w.num_tokens, H), torch.bfloat16)
        ep.ep_peer_low_latency_combine(te, r["idx"], r["h"], r["wts"], y.t, E, W, s, r["ws"])
        torch.cuda.synchronize()
        assert np.array_equal(bf16_to_u16(y.t), y_refs[s]), s
        assert y.canary_ok()
        assert ep.ep_read_status(r["ws"]) == 0


def test_peer_ll_two_ranks(ep):
    loads = [make_custom(T, 512, 4, 16, 2, seed=130 + s, mask_frac=0.05)
             for s, T in enumerate([40, 64])]
    _check_ll(ep, loads, 16, 2, 64)


def test_peer_ll_four_ranks_empty_rank(ep):
    # H = 384: 3 scale blocks per row (the per-element scale stores)
    loads = [make_custom(T, 384, 8, 32, 4, seed=140 + s) for s, T in enumerate([128, 0, 77, 128])]
    _check_ll(ep, loads, 32, 4, 128)


def test_peer_ll_eight_ranks_decode_batches(ep):
    # the low-latency workload on each of 8 ranks: 128 tokens, hidden 7168, top-8 of 256
    loads = [make_workload("ll", seed=150 + s) for s in range(8)]
    _check_ll(ep, loads, 256, 8, 128)
