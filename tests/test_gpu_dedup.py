"""GPU parity for the deduplicated path (one row per token and partition) against
the oracle, bit for bit: partition layout, payload and scales, the [rows, K]
expert lists and weights, and the combine of partition partials."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
from workloads import make_custom, make_workload, random_bf16  # noqa: E402

from gpu_path import (Guarded, bf16_to_u16, dev_u16_as_bf16, new_workspace,  # noqa: E402
                      quant_code)


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import combine_get_dispatch_05_b200 as m
    return m


def run_dedup(ep, w, quant):
    T, H, K, E, P = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
    fp8 = quant in ("fp8", "fp8_pow2")
    rows = max(T * min(P, K), 1)
    x = dev_u16_as_bf16(w.x)
    idx = torch.from_numpy(np.ascontiguousarray(w.topk_idx)).cuda()
    wts = torch.from_numpy(np.ascontiguousarray(w.topk_weights)).cuda()
    rx = Guarded((rows, H), torch.uint8 if fp8 else torch.bfloat16)
    rs = Guarded((rows, max(H // 128, 1)), torch.float32) if fp8 else None
    ri = Guarded((rows, K), torch.int32)
    rw = Guarded((rows, K), torch.float32)
    lay = ep.Layout.empty(T, P, P, P, "cuda")
    ws = new_workspace(ep, T, E, P)
    ep.ep_dispatch_dedup(x, idx, wts, E, P, quant_code(ep, quant),
                         rx.t, rs.t if fp8 else None, ri.t, rw.t, lay, ws)
    torch.cuda.synchronize()
    R = int(lay.num_recv.item())
    out = dict(R=R, lay=lay, ws=ws,
               row_of=lay.row_of.cpu().numpy(), count=lay.num_tokens_per_expert.cpu().numpy(),
               offset=lay.expert_offset.cpu().numpy(), src_of=lay.src_of[:R].cpu().numpy(),
               itp=lay.is_token_in_partition.cpu().numpy(),
               ntp=lay.num_tokens_per_partition.cpu().numpy(),
               recv_topk_idx=ri.t[:R].cpu().numpy(), recv_topk_weights=rw.t[:R].cpu().numpy())
    if fp8:
        out["recv_x"] = rx.t[:R].cpu().numpy()
        out["recv_scales"] = rs.t[:R, : H // 128].cpu().numpy()
    else:
        out["recv_x"] = bf16_to_u16(rx.t[:R])
    out["canaries_ok"] = all(g.canary_ok() for g in [rx, ri, rw] + ([rs] if fp8 else []))
    return out


CASES = [
    ("normal-300", lambda: make_workload("normal", seed=1, num_tokens=300, hidden=512)),
    ("skew-700", lambda: make_workload("skew", seed=2, num_tokens=700, hidden=256)),
    ("bf16-600", lambda: make_workload("bf16", seed=4, num_tokens=600, hidden=136)),
    ("stress-1000", lambda: make_workload("stress", seed=5, num_tokens=1000, hidden=128)),
    ("k32-dups", lambda: make_custom(70, 128, 32, 48, 6, seed=8, duplicates=True)),
    ("masked", lambda: make_custom(513, 640, 6, 64, 16, seed=10, mask_frac=0.3)),
    ("p1", lambda: make_custom(90, 128, 4, 8, 1, seed=11)),
    ("e-eq-p", lambda: make_custom(257, 256, 3, 16, 16, seed=12)),
    ("t1", lambda: make_custom(1, 128, 8, 256, 8, seed=6)),
    # fewer tokens than CTAs (some take none) and a batch with no rows at all: the
    # pipeline's end markers, one per storer warp, with nothing or little before them
    ("t5", lambda: make_custom(5, 256, 8, 64, 8, seed=17)),
    ("all-masked", lambda: make_custom(40, 256, 4, 16, 4, seed=18, mask_frac=1.0)),
    # the largest hidden size: two storers over the smallest output ring they allow
    ("h16384", lambda: make_custom(150, 16384, 8, 64, 8, seed=19, mask_frac=0.1)),
    # more than 1024 tokens: the partition layout's multi-CTA form; P = 6 and P = 5 take
    # its byte-by-byte flag and row stores, P = 32 is the most partitions it takes
    ("grid-2500", lambda: make_workload("normal", seed=3, num_tokens=2500, hidden=128)),
    ("grid-p6-3001", lambda: make_custom(3001, 128, 6, 48, 6, seed=14, mask_frac=0.1)),
    ("grid-p32-2049", lambda: make_custom(2049, 128, 8, 64, 32, seed=15, mask_frac=0.05)),
    ("p5-1025", lambda: make_custom(1025, 128, 3, 5, 5, seed=16, duplicates=True)),
]


@pytest.mark.parametrize("name,mk", CASES, ids=[c[0] for c in CASES])
def test_dispatch_dedup_parity(ep, name, mk):
    w = mk()
    quant = w.quant if w.hidden % 128 == 0 else "none"
    got = run_dedup(ep, w, quant)
    want = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, w.num_experts,
                                 w.num_partitions, quant=quant)
    lay = oracle.layout(w.topk_idx, w.num_experts, w.num_partitions)
    P = w.num_partitions
    assert got["R"] == want["num_rows"][0]
    assert np.array_equal(got["row_of"], want["prow_of"])
    assert np.array_equal(got["count"], want["part_count"])
    assert np.array_equal(got["offset"], want["part_offset"])
    assert np.array_equal(got["src_of"] // P, want["src_tok"])
    # the slot of each row is the partition whose segment holds it
    part_of_row = np.searchsorted(want["part_offset"], np.arange(got["R"]), side="right") - 1
    assert np.array_equal(got["src_of"] % P, part_of_row)
    assert np.array_equal(got["itp"], lay["is_token_in_partition"])
    assert np.array_equal(got["ntp"], lay["num_tokens_per_partition"])
    assert np.array_equal(got["recv_x"], want["recv_x"])
    if quant != "none":
        assert np.array_equal(got["recv_scales"].view(np.uint32), want["recv_scales"].view(np.uint32))
    assert np.array_equal(got["recv_topk_idx"], want["recv_topk_idx"])
    assert np.array_equal(got["recv_topk_weights"].view(np.uint32),
                          want["recv_topk_weights"].view(np.uint32))
    assert got["canaries_ok"]
    assert ep.ep_read_status(got["ws"]) == 0


@pytest.mark.parametrize("name,mk", CASES, ids=[c[0] for c in CASES])
def test_combine_dedup_parity(ep, name, mk):
    w = mk()
    got = run_dedup(ep, w, "none" if w.hidden % 128 else w.quant)
    want = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, w.num_experts,
                                 w.num_partitions, quant="none")
    R = got["R"]
    part = random_bf16(np.random.default_rng(3), (R, w.hidden), scale=2.0)
    y = torch.empty((w.num_tokens, w.hidden), dtype=torch.bfloat16, device="cuda")
    pd = dev_u16_as_bf16(part) if R else torch.empty((0, w.hidden), dtype=torch.bfloat16,
                                                     device="cuda")
    ep.ep_combine_dedup(pd, got["lay"], y, got["ws"])
    torch.cuda.synchronize()
    y_ref, st = oracle.combine_dedup(part, want["prow_of"])
    assert st == 0
    assert np.array_equal(bf16_to_u16(y), y_ref)


def test_dedup_full_size_sampled(ep):
    w = make_workload("normal", seed=4)
    got = run_dedup(ep, w, "fp8")
    lay = oracle.layout(w.topk_idx, 256, 8)
    assert got["R"] == int(lay["num_tokens_per_partition"].sum())
    assert got["R"] * 2 <= int(lay["num_recv"][0])
    rng = np.random.default_rng(2)
    for t in rng.choice(w.num_tokens, 32, replace=False):
        q, s = oracle.quantize_row(w.x[t])
        for p in range(8):
            r = got["row_of"][t, p]
            touches = bool(((w.topk_idx[t] // 32) == p).any())
            assert (r >= 0) == touches
            if r >= 0:
                assert np.array_equal(got["recv_x"][r], q)
                assert np.array_equal(got["recv_scales"][r], s)
                inside = (w.topk_idx[t] // 32) == p
                assert np.array_equal(got["recv_topk_idx"][r],
                                      np.where(inside, w.topk_idx[t] - 32 * p, -1))


def test_buffer_dedup_and_backward_methods(ep):
    w = make_workload("normal", seed=8, num_tokens=200, hidden=256)
    buf = ep.Buffer(num_experts=256, num_partitions=8, max_tokens=256)
    x = dev_u16_as_bf16(w.x)
    idx = torch.from_numpy(w.topk_idx).cuda()
    wts = torch.from_numpy(w.topk_weights).cuda()
    (q, s), ri, rw, h, ev = buf.dispatch_dedup(x, idx, wts)
    want = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, 256, 8)
    assert q.shape[0] == want["num_rows"][0]
    assert np.array_equal(q.view(torch.uint8).cpu().numpy(), want["recv_x"])
    assert np.array_equal(ri.cpu().numpy(), want["recv_topk_idx"])
    part = random_bf16(np.random.default_rng(1), (q.shape[0], 256))
    y, _ = buf.combine_dedup(dev_u16_as_bf16(part), h)
    assert np.array_equal(bf16_to_u16(y), oracle.combine_dedup(part, want["prow_of"])[0])
    # backward pair through the buffer on the per-expert layout
    _, _, _, hk, _ = buf.dispatch(x, idx, wts)
    R = int(hk.num_recv.item())
    g = random_bf16(np.random.default_rng(2), (R, 256))
    gx, gw, _ = buf.dispatch_backward(dev_u16_as_bf16(g), hk)
    lay = oracle.layout(w.topk_idx, 256, 8)
    assert gw is None
    assert np.array_equal(bf16_to_u16(gx), oracle.dispatch_backward(g, lay["row_of"])[0])
    eo = random_bf16(np.random.default_rng(3), (R, 256))
    gy = random_bf16(np.random.default_rng(4), (200, 256))
    geo, gwt, _ = buf.combine_backward(dev_u16_as_bf16(gy), dev_u16_as_bf16(eo), hk, wts)
    geo_ref, gw_ref, _ = oracle.combine_backward(gy, eo, lay["row_of"], w.topk_weights)
    assert np.array_equal(bf16_to_u16(geo), geo_ref)
    assert np.array_equal(gwt.cpu().numpy().view(np.uint32), gw_ref.view(np.uint32))
    assert buf.read_status() == 0


def test_dispatch_dedup_pow2_scales_parity(ep):
    w = make_workload("normal", seed=41, num_tokens=333, hidden=768)
    got = run_dedup(ep, w, "fp8_pow2")
    want = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, w.num_experts,
                                 w.num_partitions, quant="fp8_pow2")
    assert got["R"] == want["num_rows"][0]
    assert np.array_equal(got["recv_x"], want["recv_x"])
    assert np.array_equal(got["recv_scales"].view(np.uint32), want["recv_scales"].view(np.uint32))
    assert got["canaries_ok"]


def test_dispatch_dedup_block_major_pow2_scales(ep):
    # deduplicated rows with power-of-two scales stored block-major: scale of row r,
    # block b at [b * ld + r], ld = T * min(P, K) rounded up to 4
    w = make_custom(301, 640, 6, 64, 16, seed=13, mask_frac=0.1)
    T, H, K, E, P = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
    rows = T * min(P, K)
    nb, ld = H // 128, ep.scales_ld(rows)
    x = dev_u16_as_bf16(w.x)
    idx = torch.from_numpy(np.ascontiguousarray(w.topk_idx)).cuda()
    wts = torch.from_numpy(np.ascontiguousarray(w.topk_weights)).cuda()
    rq = torch.empty((rows, H), dtype=torch.uint8, device="cuda")
    rs = torch.full((nb * ld,), float("nan"), dtype=torch.float32, device="cuda")
    ri = torch.empty((rows, K), dtype=torch.int32, device="cuda")
    rw = torch.empty((rows, K), dtype=torch.float32, device="cuda")
    lay = ep.Layout.empty(T, P, P, P, "cuda")
    ws = new_workspace(ep, T, E, P)
    ep.ep_dispatch_dedup(x, idx, wts, E, P,
                         ep.EP_QUANT_FP8_E4M3_1X128_POW2 | ep.EP_QUANT_SCALES_MN_MAJOR,
                         rq, rs, ri, rw, lay, ws)
    torch.cuda.synchronize()
    want = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, E, P, quant="fp8_pow2")
    R = int(want["num_rows"][0])
    got = rs.view(nb, ld).cpu().numpy()
    assert np.array_equal(got[:, :R].T.view(np.uint32), want["recv_scales"].view(np.uint32))
    assert np.all(np.isnan(got[:, R:]))
    assert np.array_equal(rq[:R].cpu().numpy(), want["recv_x"])
    assert ep.ep_read_status(ws) == 0


def test_dedup_layout_skips_and_reports_out_of_range_ids(ep):
    # ids outside [-1, E) count as masked in the deduplicated layout too, and are reported
    w = make_custom(1500, 128, 8, 64, 8, seed=17)
    bad = w.topk_idx.copy()
    bad[3, 2], bad[1200, 0], bad[700, 7] = 64, -5, 1000
    T, K, E, P = w.num_tokens, w.num_topk, w.num_experts, w.num_partitions
    idx = torch.from_numpy(bad).cuda()
    lay = ep.Layout.empty(T, P, P, P, "cuda")
    ws = new_workspace(ep, T, E, P)
    ep.ep_get_dispatch_layout_dedup(idx, E, P, lay, ws)
    torch.cuda.synchronize()
    clean = np.where((bad >= 0) & (bad < E), bad, -1)
    want = oracle.dispatch_dedup(w.x, clean, w.topk_weights, E, P, quant="none")
    assert np.array_equal(lay.row_of.cpu().numpy(), want["prow_of"])
    assert np.array_equal(lay.expert_offset.cpu().numpy(), want["part_offset"])
    assert ep.ep_read_status(ws) == ep.EP_DEV_INDEX_RANGE
