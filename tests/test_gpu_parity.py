"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact comparisons throughout: layout arrays, E4M3 payload bytes, fp32
scale bits, BF16 copies, and combine outputs (the kernel keeps the oracle's
fixed k-order fmaf chain).  Sizes span several layout chunks (256 tokens) and
ragged tails; edge cases cover empty batches, single tokens, all-masked
tokens, duplicate experts, out-of-range ids, K = 1 / 32, E = 1 and the scale
paths with H/128 blocks not a multiple of 4.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
from workloads import make_custom, make_workload, random_bf16  # noqa: E402

from gpu_path import (bf16_to_u16, dev_u16_as_bf16, gpu_combine, gpu_dispatch, gpu_layout,  # noqa: E402
                      layout_numpy, new_workspace, torch_identity_expert)


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import combine_get_dispatch_05_b200 as m
    return m


LAYOUT_KEYS = ("num_tokens_per_expert", "num_tokens_per_partition", "is_token_in_partition",
               "expert_offset", "row_of", "src_of", "num_recv")


def _assert_layout(got, want):
    for k in LAYOUT_KEYS:
        assert np.array_equal(got[k], want[k]), k


def _cases():
    yield "normal-300", make_workload("normal", seed=1, num_tokens=300, hidden=512)
    yield "skew-700", make_workload("skew", seed=2, num_tokens=700, hidden=256)
    yield "ll-128", make_workload("ll", seed=3, hidden=384)
    yield "bf16-600", make_workload("bf16", seed=4, num_tokens=600, hidden=136)
    yield "stress-1000", make_workload("stress", seed=5, num_tokens=1000, hidden=128)
    yield "t1", make_custom(1, 128, 8, 256, 8, seed=6)
    yield "k1", make_custom(257, 256, 1, 16, 4, seed=7)
    yield "k32-dups", make_custom(70, 128, 32, 48, 6, seed=8, duplicates=True)
    yield "e1", make_custom(33, 128, 2, 1, 1, seed=9, duplicates=True)
    yield "masked", make_custom(513, 640, 6, 64, 16, seed=10, mask_frac=0.3)
    yield "hot", make_custom(800, 128, 4, 32, 8, seed=11, hot_expert=5)
    yield "e4096", make_custom(300, 128, 8, 4096, 64, seed=12)
    # the largest hidden size the calls take: one dispatch CTA per SM, the fewest
    # staged rows
    yield "h16384", make_custom(150, 16384, 8, 64, 8, seed=13, mask_frac=0.1)


CASES = list(_cases())


@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_layout_parity(ep, name, w):
    lay, ws = gpu_layout(ep, w.topk_idx, w.num_experts, w.num_partitions)
    got = layout_numpy(lay, w.num_tokens, w.num_topk)
    want = oracle.layout(w.topk_idx, w.num_experts, w.num_partitions)
    _assert_layout(got, want)
    assert ep.ep_read_status(ws) == 0


@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_dispatch_parity(ep, name, w):
    quant = w.quant if w.hidden % 128 == 0 else "none"
    got, _ = gpu_dispatch(ep, w, quant=quant)
    want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, w.num_experts, w.num_partitions,
                           quant=quant)
    _assert_layout(got, want)
    assert np.array_equal(got["recv_x"], want["recv_x"])
    if quant == "fp8":
        assert np.array_equal(got["recv_scales"].view(np.uint32),
                              want["recv_scales"].view(np.uint32))
    assert np.array_equal(got["recv_topk_idx"], want["recv_topk_idx"])
    assert np.array_equal(got["recv_topk_weights"].view(np.uint32),
                          want["recv_topk_weights"].view(np.uint32))
    assert got["canaries_ok"]


@pytest.mark.parametrize("name,w", CASES, ids=[c[0] for c in CASES])
def test_combine_parity_random_expert_out(ep, name, w):
    rng = np.random.default_rng(100)
    lay, ws = gpu_layout(ep, w.topk_idx, w.num_experts, w.num_partitions)
    want_lay = oracle.layout(w.topk_idx, w.num_experts, w.num_partitions)
    R = int(want_lay["num_recv"][0])
    H = w.hidden if w.hidden % 8 == 0 else 128
    eo = random_bf16(rng, (R, H), scale=3.0)
    y, canary = gpu_combine(ep, eo, lay, w.topk_weights, ws)
    y_ref, st = oracle.combine(eo, want_lay["row_of"], w.topk_weights)
    assert st == 0 and canary
    assert np.array_equal(y, y_ref)


@pytest.mark.parametrize("name", ["normal", "skew", "bf16"])
def test_chain_dispatch_identity_combine(ep, name):
    w = make_workload(name, seed=21, num_tokens=520, hidden=1024 if name != "bf16" else 264)
    got, st = gpu_dispatch(ep, w)
    if w.quant == "fp8":
        eo = torch_identity_expert(st["recv_x"], st["recv_s"])
    else:
        eo = st["recv_x"]
    y = torch.empty((w.num_tokens, w.hidden), dtype=torch.bfloat16, device="cuda")
    ep.ep_combine(eo, st["layout"], st["wts"], y, st["ws"])
    want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, w.num_experts, w.num_partitions,
                           quant=w.quant)
    eo_ref = oracle.identity_expert(want["recv_x"], want.get("recv_scales"), quant=w.quant)
    y_ref, _ = oracle.combine(eo_ref, want["row_of"], w.topk_weights)
    assert np.array_equal(bf16_to_u16(y), y_ref)


def test_dispatch_is_deterministic(ep):
    w = make_workload("skew", seed=3, num_tokens=1500, hidden=512)
    a, _ = gpu_dispatch(ep, w)
    b, _ = gpu_dispatch(ep, w)
    for k in ("row_of", "src_of", "recv_x", "recv_scales"):
        assert np.array_equal(a[k], b[k]), k


def test_empty_batch(ep):
    w = make_custom(0, 128, 8, 32, 4)
    got, st = gpu_dispatch(ep, w)
    assert got["num_recv"][0] == 0
    assert np.all(got["expert_offset"] == 0) and np.all(got["num_tokens_per_expert"] == 0)
    y = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    ep.ep_combine(torch.empty((0, 128), dtype=torch.bfloat16, device="cuda"), st["layout"],
                  st["wts"], y, st["ws"])


def test_workspace_reuse_across_batch_sizes(ep):
    # one workspace sized for the largest batch serves smaller, ragged ones
    ws = new_workspace(ep, 2000, 256, 8)
    for T in (2000, 1999, 257, 3, 1024):
        w = make_workload("normal", seed=T, num_tokens=T, hidden=128)
        got, _ = gpu_dispatch(ep, w, workspace=ws)
        want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 256, 8)
        _assert_layout(got, want)
        assert np.array_equal(got["recv_x"], want["recv_x"])


def test_out_of_range_ids_are_skipped_and_reported(ep):
    w = make_custom(300, 256, 4, 16, 4, seed=13)
    w.topk_idx[5, 1] = 16
    w.topk_idx[77, 3] = -9
    w.topk_idx[299, 0] = 1 << 40
    got, st = gpu_dispatch(ep, w)
    want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 16, 4)
    assert want["status"] & oracle.INDEX_RANGE
    _assert_layout(got, want)
    assert np.array_equal(got["recv_x"], want["recv_x"])
    assert ep.ep_read_status(st["ws"]) & ep.EP_DEV_INDEX_RANGE
    assert ep.ep_read_status(st["ws"]) == 0  # read clears


def test_combine_row_outside_buffer_is_reported(ep):
    rng = np.random.default_rng(1)
    T, K, H = 40, 3, 256
    eo = random_bf16(rng, (10, H))
    lay = ep.Layout.empty(T, K, 4, 1, "cuda")
    row_of = rng.integers(-1, 10, size=(T, K)).astype(np.int32)
    row_of[7, 2] = 10  # one past the end
    lay.row_of.copy_(torch.from_numpy(row_of))
    w = rng.standard_normal((T, K)).astype(np.float32)
    ws = new_workspace(ep, T, 4, 1)
    y, ok = gpu_combine(ep, eo, lay, w, ws)
    y_ref, st = oracle.combine(eo, row_of, w)
    assert st & oracle.INDEX_RANGE and ok
    assert np.array_equal(y, y_ref)
    assert ep.ep_read_status(ws) & ep.EP_DEV_INDEX_RANGE


# ---------------------------------------------------------------- low latency --

def _ll_gpu(ep, w, cap):
    T, H, K, E = w.num_tokens, w.hidden, w.num_topk, w.num_experts
    x = torch.from_numpy(w.x.view(np.int16)).cuda().view(torch.bfloat16)
    idx = torch.from_numpy(w.topk_idx).cuda()
    recv_x = torch.full((E, cap, H), 0xA5, dtype=torch.uint8, device="cuda")
    recv_s = torch.full((E, cap, H // 128), -1.0, dtype=torch.float32, device="cuda")
    count = torch.empty(E, dtype=torch.int32, device="cuda")
    h = ep.LowLatencyHandle.empty(T, K, E, cap, "cuda")
    h.src_of.fill_(-1)
    ws = new_workspace(ep, 1, E, 1)
    ep.ep_low_latency_dispatch(x, idx, cap, E, recv_x, recv_s, count, h, ws)
    torch.cuda.synchronize()
    return dict(recv_x=recv_x.cpu().numpy(), recv_scales=recv_s.cpu().numpy(),
                recv_expert_count=count.cpu().numpy(), ll_row_of=h.row_of.cpu().numpy(),
                ll_src_of=h.src_of.cpu().numpy()), (h, ws, recv_x, recv_s)


LL_CASES = [
    ("ll", make_workload("ll", seed=0, hidden=512), 128),
    ("ll-7168", make_workload("ll", seed=1, num_tokens=40), 128),
    ("ll-h384", make_workload("ll", seed=2, num_tokens=97, hidden=384), 100),
    ("ll-masked", make_custom(64, 256, 6, 32, 1, seed=3, mask_frac=0.2), 64),
    ("ll-dups-overflow", make_custom(20, 128, 4, 3, 1, seed=4, duplicates=True), 20),
    ("ll-t1", make_custom(1, 128, 8, 256, 1, seed=5), 128),
    ("ll-e2048", make_custom(300, 256, 8, 2048, 1, seed=6), 300),
]


@pytest.mark.parametrize("name,w,cap", LL_CASES, ids=[c[0] for c in LL_CASES])
def test_ll_dispatch_parity(ep, name, w, cap):
    got, (h, ws, _, _) = _ll_gpu(ep, w, cap)
    want = oracle.ll_dispatch(w.x, w.topk_idx, w.num_experts, cap, fill=0xA5)
    assert np.array_equal(got["recv_expert_count"], want["recv_expert_count"])
    assert np.array_equal(got["ll_row_of"], want["ll_row_of"])
    # the whole padded tensor: written slots bit-exact, unwritten slots untouched
    assert np.array_equal(got["recv_x"], want["recv_x"])
    assert np.array_equal(got["recv_scales"].view(np.uint32), want["recv_scales"].view(np.uint32))
    assert np.array_equal(got["ll_src_of"], want["ll_src_of"])
    bits = ep.ep_read_status(ws)
    assert bool(bits & ep.EP_DEV_CAPACITY) == bool(want["status"] & oracle.CAPACITY)


@pytest.mark.parametrize("name,w,cap", LL_CASES, ids=[c[0] for c in LL_CASES])
def test_ll_combine_parity(ep, name, w, cap):
    got, (h, ws, _, _) = _ll_gpu(ep, w, cap)
    rng = np.random.default_rng(9)
    eo = random_bf16(rng, (w.num_experts, cap, w.hidden))
    y = torch.empty((w.num_tokens, w.hidden), dtype=torch.bfloat16, device="cuda")
    eo_d = torch.from_numpy(eo.view(np.int16)).cuda().view(torch.bfloat16)
    wts = torch.from_numpy(w.topk_weights).cuda()
    ep.ep_low_latency_combine(eo_d, h, wts, y, ws)
    want = oracle.ll_dispatch(w.x, w.topk_idx, w.num_experts, cap)
    y_ref, _ = oracle.ll_combine(eo, want["ll_row_of"], w.topk_weights)
    assert np.array_equal(bf16_to_u16(y), y_ref)


def test_ll_equals_normal(ep):
    w = make_workload("ll", seed=7, hidden=1024)
    cap = w.num_max_tokens
    ll, (h, ws, recv_q, recv_s) = _ll_gpu(ep, w, cap)
    nd, st = gpu_dispatch(ep, w)
    off = nd["expert_offset"]
    for e in range(w.num_experts):
        n = ll["recv_expert_count"][e]
        assert np.array_equal(ll["recv_x"][e, :n], nd["recv_x"][off[e]:off[e] + n])
    # LL combine == normal combine on identity experts, bit for bit
    y_n = torch.empty((w.num_tokens, w.hidden), dtype=torch.bfloat16, device="cuda")
    ep.ep_combine(torch_identity_expert(st["recv_x"], st["recv_s"]), st["layout"], st["wts"], y_n,
                  st["ws"])
    y_l = torch.empty_like(y_n)
    ep.ep_low_latency_combine(torch_identity_expert(recv_q, recv_s), h, st["wts"], y_l, ws)
    assert torch.equal(y_n.view(torch.int16), y_l.view(torch.int16))


# ----------------------------------------------------- status / bounded waits --

def test_bounded_wait_gives_up_and_context_survives(ep):
    ws = new_workspace(ep, 1, 1, 1)
    ep.ep_debug_wait_probe(2_000_000, ws)  # 2 ms
    assert ep.ep_read_status(ws) & ep.EP_DEV_TIMEOUT
    # the context is still usable
    w = make_custom(50, 128, 2, 8, 2, seed=1)
    got, _ = gpu_dispatch(ep, w)
    want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 8, 2)
    assert np.array_equal(got["recv_x"], want["recv_x"])


# ------------------------------------------------------------------ Buffer API --

def test_buffer_api_matches_pages_call_shapes(ep):
    w = make_workload("normal", seed=2, num_tokens=333, hidden=256)
    buf = ep.Buffer(num_experts=256, num_partitions=8, max_tokens=512)
    x = torch.from_numpy(w.x.view(np.int16)).cuda().view(torch.bfloat16)
    idx = torch.from_numpy(w.topk_idx).cuda()
    wts = torch.from_numpy(w.topk_weights).cuda()
    recv_x, recv_topk_idx, recv_topk_weights, handle, event = buf.dispatch(x, idx, wts, 256)
    event.synchronize()
    want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 256, 8)
    q, s = recv_x
    assert q.dtype == torch.float8_e4m3fn and q.shape[0] == int(want["num_recv"][0])
    assert np.array_equal(q.view(torch.uint8).cpu().numpy(), want["recv_x"])
    assert np.array_equal(recv_topk_idx.cpu().numpy(), want["recv_topk_idx"])
    y, ev = buf.combine(torch_identity_expert(q, s), handle, wts)
    eo_ref = oracle.identity_expert(want["recv_x"], want["recv_scales"])
    y_ref, _ = oracle.combine(eo_ref, want["row_of"], w.topk_weights)
    assert np.array_equal(bf16_to_u16(y), y_ref)
    (rq, rs), cnt, lh, ev, hook = buf.low_latency_dispatch(x[:128], idx[:128], 128, 256)
    hook()
    assert np.array_equal(cnt.cpu().numpy(),
                          oracle.layout(w.topk_idx[:128], 256, 8)["num_tokens_per_expert"])
    assert buf.read_status() == 0


POW2_CASES = [c for c in CASES if c[0] in ("normal-300", "masked", "k32-dups", "e4096", "t1")]


@pytest.mark.parametrize("name,w", POW2_CASES, ids=[c[0] for c in POW2_CASES])
def test_dispatch_pow2_scales_parity(ep, name, w):
    got, _ = gpu_dispatch(ep, w, quant="fp8_pow2")
    want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, w.num_experts, w.num_partitions,
                           quant="fp8_pow2")
    _assert_layout(got, want)
    assert np.array_equal(got["recv_x"], want["recv_x"])
    assert np.array_equal(got["recv_scales"].view(np.uint32), want["recv_scales"].view(np.uint32))
    assert np.all((got["recv_scales"].view(np.uint32) & 0x007FFFFF) == 0)  # exponent only
    assert got["canaries_ok"]


def test_pow2_scales_on_extreme_blocks(ep):
    # blocks whose amax sits exactly on, just above and just below 448 * 2^n, and
    # all-zero / subnormal-only blocks (the 1e-4 floor)
    f = np.zeros((4, 1024), np.float32)
    f[0, :128] = 448.0
    f[0, 128:256] = np.float32(448.0 * 2 ** -3)
    f[0, 256:384] = 449.0
    f[0, 384:512] = 447.0
    f[1, :128] = 1e-40
    f[2] = np.linspace(-3000, 3000, 1024, dtype=np.float32)
    f[3, ::7] = -2.0 ** 100
    x = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    w = make_custom(4, 1024, 2, 8, 2, seed=30)
    w.x[:] = x
    got, _ = gpu_dispatch(ep, w, quant="fp8_pow2")
    want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 8, 2, quant="fp8_pow2")
    assert np.array_equal(got["recv_x"], want["recv_x"])
    assert np.array_equal(got["recv_scales"].view(np.uint32), want["recv_scales"].view(np.uint32))


@pytest.mark.parametrize("T,K,E,P", [(40000, 8, 256, 8), (65536, 8, 256, 8), (16384, 32, 64, 8)])
def test_layout_parity_large_batches(ep, T, K, E, P):
    # batches whose ids no longer fit one cluster's shared memory take the
    # cooperative-grid layout; those just below take the cluster with large chunks
    w = make_custom(T, 128, K, E, P, seed=T + K, mask_frac=0.05)
    lay, ws = gpu_layout(ep, w.topk_idx, E, P)
    got = layout_numpy(lay, T, K)
    _assert_layout(got, oracle.layout(w.topk_idx, E, P))
    assert ep.ep_read_status(ws) == 0


def test_dispatch_ticket_words_return_to_zero(ep):
    # the dispatch kernels hand tokens out from a counter in the workspace header
    # (bytes 16..23); the last CTA to finish re-zeroes it for the next call
    ws = new_workspace(ep, 700, 256, 8)
    for name, T, H in (("normal", 700, 256), ("bf16", 333, 136), ("normal", 5, 128)):
        w = make_workload(name, seed=T, num_tokens=T, hidden=H)
        quant = w.quant if H % 128 == 0 else "none"
        got, _ = gpu_dispatch(ep, w, workspace=ws, quant=quant)
        want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, w.num_experts, w.num_partitions,
                               quant=quant)
        assert np.array_equal(got["recv_x"], want["recv_x"])
        assert np.array_equal(got["src_of"], want["src_of"])
        assert ws[16:24].cpu().numpy().tolist() == [0] * 8


def test_quantiser_quotients_on_exact_midpoints(ep):
    # Blocks whose scale s = c * 2^k has few significant bits (c in 1, 3, 5) and whose
    # elements are E4M3 values and midpoints times s, all exact in BF16: x / s is then
    # exactly an E4M3 value or a tie, so a quotient off by one ulp would change the
    # code.  The kernel's quotient (Markstein correction step) must give the oracle's
    # IEEE division result everywhere.
    rng = np.random.default_rng(77)
    codes = np.arange(0x7F)
    E_, m_ = codes >> 3, codes & 7
    vals = np.where(E_ == 0, m_ * 2.0 ** -9, (1 + m_ / 8.0) * 2.0 ** (E_ - 7))
    grid = np.unique(np.concatenate([vals, (vals[:-1] + vals[1:]) / 2]))
    T, H = 96, 1024
    f = np.zeros((T, H), np.float64)
    for t in range(T):
        for b in range(H // 128):
            c = rng.choice([1.0, 3.0, 5.0])
            s = c * 2.0 ** int(rng.integers(-20, 13))
            blk = rng.choice(grid, 128) * s * np.where(rng.random(128) < 0.5, -1.0, 1.0)
            blk[rng.integers(0, 128)] = 448.0 * s * (1 if rng.random() < 0.5 else -1)
            f[t, b * 128:(b + 1) * 128] = blk
    x32 = f.astype(np.float32)
    x = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal((x.astype(np.uint32) << 16).view(np.float32), x32)  # exact in BF16
    w = make_custom(T, H, 2, 8, 2, seed=78)
    w.x[:] = x
    for quant in ("fp8", "fp8_pow2"):
        got, _ = gpu_dispatch(ep, w, quant=quant)
        want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 8, 2, quant=quant)
        assert np.array_equal(got["recv_x"], want["recv_x"]), quant
        assert np.array_equal(got["recv_scales"].view(np.uint32), want["recv_scales"].view(np.uint32))


@pytest.mark.parametrize("quant,name,mk", [
    ("fp8", "normal-300", lambda: make_workload("normal", seed=1, num_tokens=300, hidden=512)),
    ("fp8_pow2", "masked", lambda: make_custom(513, 640, 6, 64, 16, seed=10, mask_frac=0.3)),
    ("fp8", "t1", lambda: make_custom(1, 128, 8, 256, 8, seed=6)),
])
def test_dispatch_block_major_scales(ep, quant, name, mk):
    # EP_QUANT_SCALES_MN_MAJOR: the scale of row r, block b at [b * ld + r],
    # ld = T*K rounded up to 4; entries past the received rows are not written
    w = mk()
    T, H, K, E, P = w.num_tokens, w.hidden, w.num_topk, w.num_experts, w.num_partitions
    nb, ld = H // 128, ep.scales_ld(T * K)
    x = dev_u16_as_bf16(w.x)
    idx = torch.from_numpy(np.ascontiguousarray(w.topk_idx)).cuda()
    wts = torch.from_numpy(np.ascontiguousarray(w.topk_weights)).cuda()
    rq = torch.empty((T * K, H), dtype=torch.uint8, device="cuda")
    rs = torch.full((nb * ld + 4,), float("nan"), dtype=torch.float32, device="cuda")
    ri = torch.empty(T * K, dtype=torch.int32, device="cuda")
    rw = torch.empty(T * K, dtype=torch.float32, device="cuda")
    lay = ep.Layout.empty(T, K, E, P, "cuda")
    ws = new_workspace(ep, T, E, P)
    base = {"fp8": ep.EP_QUANT_FP8_E4M3_1X128, "fp8_pow2": ep.EP_QUANT_FP8_E4M3_1X128_POW2}[quant]
    ep.ep_dispatch(x, idx, wts, E, P, base | ep.EP_QUANT_SCALES_MN_MAJOR, rq, rs, ri, rw, lay, ws)
    torch.cuda.synchronize()
    want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, E, P, quant=quant)
    R = int(want["num_recv"][0])
    got = rs[:nb * ld].view(nb, ld).cpu().numpy()
    assert np.array_equal(got[:, :R].T.view(np.uint32), want["recv_scales"].view(np.uint32))
    assert np.all(np.isnan(got[:, R:])) and bool(torch.isnan(rs[nb * ld:]).all())
    assert np.array_equal(rq[:R].cpu().numpy(), want["recv_x"])
    assert ep.ep_read_status(ws) == 0


def test_buffer_block_major_scales_view(ep):
    w = make_workload("normal", seed=3, num_tokens=200, hidden=256)
    buf = ep.Buffer(num_experts=256, num_partitions=8, max_tokens=256)
    x = dev_u16_as_bf16(w.x)
    idx = torch.from_numpy(w.topk_idx).cuda()
    wts = torch.from_numpy(w.topk_weights).cuda()
    (q1, s1), *_ = buf.dispatch(x, idx, wts, scales_mn_major=True)
    (q0, s0), *_ = buf.dispatch(x, idx, wts)
    assert s1.shape == s0.shape and s1.stride(0) == 1  # an [R, H/128] view, block-major
    assert torch.equal(s1, s0) and torch.equal(q1.view(torch.uint8), q0.view(torch.uint8))


def test_layout_too_large_batch_is_a_shape_error(ep):
    # each SM keeps its chunk of ids in shared memory: far beyond that the call
    # returns EP_ERR_SHAPE before launching anything
    T, K, E, P = 1 << 21, 8, 256, 8
    idx = torch.zeros((T, K), dtype=torch.int64, device="cuda")
    lay = ep.Layout.empty(T, K, E, P, "cuda")
    ws = new_workspace(ep, 1, E, P)
    with pytest.raises(ep.EpError) as err:
        ep.ep_get_dispatch_layout(idx, E, P, lay, torch.empty(ep.ep_workspace_bytes(T, E, P),
                                                             dtype=torch.uint8, device="cuda"))
    assert err.value.status == ep.EP_ERR_SHAPE
    assert ep.ep_read_status(ws) == 0


class _FakeGroup:
    """Stands in for a process group of 8 ranks (only size() is read)."""

    def size(self):
        return 8


def test_buffer_pages_constructor_and_growing_workspace(ep):
    # Buffer(group, num_nvl_bytes, num_rdma_bytes, low_latency_mode) as on the pages;
    # num_experts comes with the first dispatch; a larger batch grows the workspace
    buf = ep.Buffer(_FakeGroup(), int(1e9), 0, False)
    assert buf.num_partitions == 8 and buf.num_experts is None
    for T in (100, 700):
        w = make_workload("normal", seed=T, num_tokens=T, hidden=256)
        x = dev_u16_as_bf16(w.x)
        idx = torch.from_numpy(w.topk_idx).cuda()
        wts = torch.from_numpy(w.topk_weights).cuda()
        (q, s), ri, rw, handle, ev = buf.dispatch(x, idx, wts, 256)
        ev.synchronize()
        want = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 256, 8)
        assert np.array_equal(q.view(torch.uint8).cpu().numpy(), want["recv_x"])
        assert np.array_equal(s.cpu().numpy().view(np.uint32), want["recv_scales"].view(np.uint32))
        assert buf.max_tokens >= T
    with pytest.raises(ValueError):
        buf.dispatch(x, idx, wts, 128)  # the buffer's experts are fixed by now
    assert buf.read_status() == 0
