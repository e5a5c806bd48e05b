"""Pins for the oracle's layout, dispatch, combine and low-latency steps.

Pinned against brute force on tiny inputs (Python loops over dicts, written
differently from the C loops), library routines (``numpy.argsort`` with a
stable sort), float64 exact sums with the fmaf-chain error bound, and the
invariants the method fixes: per-expert counts sum to T*K minus masked
slots; dispatch then combine with identity experts and weights summing to one
gives x back within FP8 error; the low-latency padded layout agrees with the
normal layout row for row.
"""
from collections import Counter, defaultdict

import numpy as np
import pytest

import oracle
from workloads import f32_from_bf16_bits, make_custom, make_workload, random_bf16


def _brute_layout(idx, E, P):
    T, K = idx.shape
    epp = E // P
    pairs = defaultdict(list)
    cnt = Counter()
    parts = [set() for _ in range(P)]
    bad = False
    for t in range(T):
        for k in range(K):
            e = int(idx[t, k])
            if e == -1:
                continue
            if not 0 <= e < E:
                bad = True
                continue
            pairs[e].append((t, k))
            cnt[e] += 1
            parts[e // epp].add(t)
    rows = {}
    r = 0
    for e in range(E):
        for tk in pairs[e]:  # already (t, k)-ascending
            rows[tk] = r
            r += 1
    return cnt, [len(s) for s in parts], rows, r, bad


def _tiny_cases():
    rng = np.random.default_rng(1)
    for case in range(60):
        T = int(rng.integers(0, 9))
        K = int(rng.integers(1, 4))
        P = int(rng.choice([1, 2, 4]))
        E = P * int(rng.integers(1, 3))
        idx = rng.integers(-1, E, size=(T, K)).astype(np.int64)
        if case % 7 == 3 and T:
            idx[0, 0] = E + 3  # out of range
        if case % 11 == 5 and T:
            idx[-1, -1] = -7
        yield idx, E, P


def test_layout_bruteforce_tiny():
    for idx, E, P in _tiny_cases():
        T, K = idx.shape
        lay = oracle.layout(idx, E, P)
        cnt, pcnt, rows, R, bad = _brute_layout(idx, E, P)
        assert lay["num_recv"][0] == R
        assert list(lay["num_tokens_per_expert"]) == [cnt[e] for e in range(E)]
        assert list(lay["num_tokens_per_partition"]) == pcnt
        assert bool(lay["status"] & oracle.INDEX_RANGE) == bad
        for t in range(T):
            for k in range(K):
                want = rows.get((t, k), -1)
                assert lay["row_of"][t, k] == want
                if want >= 0:
                    assert lay["src_of"][want] == t * K + k
        off = np.concatenate([[0], np.cumsum([cnt[e] for e in range(E)])])
        assert np.array_equal(lay["expert_offset"], off)


@pytest.mark.parametrize("name", ["normal", "skew", "ll"])
def test_layout_matches_stable_argsort(name):
    w = make_workload(name, seed=0, hidden=128)
    lay = oracle.layout(w.topk_idx, w.num_experts, w.num_partitions)
    flat = w.topk_idx.reshape(-1)
    valid = np.nonzero(flat >= 0)[0]
    order = valid[np.argsort(flat[valid], kind="stable")]
    R = int(lay["num_recv"][0])
    assert R == valid.size == w.num_tokens * w.num_topk - int((flat == -1).sum())
    assert np.array_equal(lay["src_of"], order)
    ro = lay["row_of"].reshape(-1)
    assert np.array_equal(ro[order], np.arange(R))
    assert np.all(ro[flat == -1] == -1)
    # counts sum to T*K minus masked slots; offsets end at R
    assert lay["num_tokens_per_expert"].sum() == R == lay["expert_offset"][-1]
    # inside every expert segment src_of increases (token, then slot order)
    off = lay["expert_offset"]
    for e in range(w.num_experts):
        seg = lay["src_of"][off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.all(flat[seg] == e)
    # partitions: distinct tokens touching each partition
    epp = w.experts_per_partition
    itp = lay["is_token_in_partition"]
    for p in range(w.num_partitions):
        touch = ((w.topk_idx >= p * epp) & (w.topk_idx < (p + 1) * epp)).any(axis=1)
        assert np.array_equal(itp[:, p].astype(bool), touch)
        assert lay["num_tokens_per_partition"][p] == touch.sum()
        assert touch.sum() <= lay["num_tokens_per_expert"][p * epp:(p + 1) * epp].sum()


def test_partition_rows_are_contiguous_slices():
    w = make_workload("normal", seed=1, num_tokens=300, hidden=128)
    d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, w.num_experts, w.num_partitions)
    epp = w.experts_per_partition
    off = d["expert_offset"]
    for p in range(w.num_partitions):
        lo, hi = off[p * epp], off[(p + 1) * epp]
        experts = w.topk_idx.reshape(-1)[d["src_of"][lo:hi]]
        assert np.all((experts >= p * epp) & (experts < (p + 1) * epp))
        # recv_topk_idx is the local expert id inside the partition
        assert np.array_equal(d["recv_topk_idx"][lo:hi], experts - p * epp)


def test_dispatch_rows_are_quantised_source_rows():
    w = make_custom(37, 384, 3, 8, 2, seed=4, mask_frac=0.1)
    d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 8, 2)
    q, s = oracle.quantize_rows(w.x)
    R = int(d["num_recv"][0])
    for r in range(R):
        t, k = divmod(int(d["src_of"][r]), 3)
        assert np.array_equal(d["recv_x"][r], q[t])
        assert np.array_equal(d["recv_scales"][r], s[t])
        assert d["recv_topk_weights"][r] == w.topk_weights[t, k]


def test_bf16_dispatch_is_bit_copy():
    w = make_custom(41, 64, 4, 12, 3, seed=2, quant="none", mask_frac=0.05)
    d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 12, 3, quant="none")
    src_t = d["src_of"] // 4
    assert np.array_equal(d["recv_x"], w.x[src_t])


def _exact_combine(eo, row_of, wts):
    T, K = row_of.shape
    e = f32_from_bf16_bits(eo).astype(np.float64)
    y = np.zeros((T, eo.shape[1]))
    mag = np.zeros_like(y)
    for t in range(T):
        for k in range(K):
            r = row_of[t, k]
            if r >= 0:
                y[t] += float(wts[t, k]) * e[r]
                mag[t] += abs(float(wts[t, k])) * np.abs(e[r])
    return y, mag


def test_combine_vs_float64_bound():
    rng = np.random.default_rng(8)
    for K in (1, 2, 5, 8):
        T, H, R = 23, 256, 40
        eo = random_bf16(rng, (R, H))
        row_of = rng.integers(-1, R, size=(T, K)).astype(np.int32)
        w = rng.standard_normal((T, K)).astype(np.float32)
        y, st = oracle.combine(eo, row_of, w)
        assert st == 0
        exact, mag = _exact_combine(eo, row_of, w)
        yf = f32_from_bf16_bits(y).astype(np.float64)
        # fmaf chain: each step rounds once -> <= K * 2^-24 * sum|w e|, then BF16 half ulp
        half_ulp = np.abs(exact) * 2.0 ** -8 + 2.0 ** -133
        assert np.all(np.abs(yf - exact) <= K * 2.0 ** -24 * mag * 1.01 + half_ulp * 1.01 + 1e-30)


def test_combine_special_cases():
    rng = np.random.default_rng(2)
    eo = random_bf16(rng, (6, 128))
    # single slot with weight 1: y is that expert row exactly
    row_of = np.array([[3], [0], [5]], np.int32)
    y, _ = oracle.combine(eo, row_of, np.ones((3, 1), np.float32))
    assert np.array_equal(y, eo[[3, 0, 5]])
    # weight -1 flips the sign bit
    y, _ = oracle.combine(eo, row_of, -np.ones((3, 1), np.float32))
    assert np.array_equal(y, eo[[3, 0, 5]] ^ 0x8000)
    # all slots masked: +0 (bit pattern 0), whatever the weights say
    y, _ = oracle.combine(eo, np.full((2, 4), -1, np.int32), np.full((2, 4), 7.0, np.float32))
    assert np.all(y == 0)
    # a row outside the expert-output buffer is skipped and reported
    y, st = oracle.combine(eo, np.array([[9, 1]], np.int32), np.ones((1, 2), np.float32))
    assert st & oracle.INDEX_RANGE and np.array_equal(y, eo[[1]])


def _bf16_of(v):
    return int(np.array([v], np.float32).view(np.uint32)[0] >> 16)


def test_combine_k_order_is_ascending():
    # terms 1, 2^-8, 2^-24, 2^-24 (expert rows all 1.0, the weights carry the
    # values).  k ascending: 1 + 2^-8, then each 2^-24 is a float32 half-ulp
    # tie that rounds back to 1 + 2^-8; BF16 then ties to even -> 1.0.
    # Reversed: 2^-23 + 2^-8 + 1 = 1 + 2^-8 + 2^-23 exactly -> BF16 1 + 2^-7.
    eo = np.full((4, 128), 0x3F80, np.uint16)
    w = np.array([[1.0, 2.0 ** -8, 2.0 ** -24, 2.0 ** -24]], np.float32)
    y, _ = oracle.combine(eo, np.array([[0, 1, 2, 3]], np.int32), w)
    assert y[0, 0] == 0x3F80
    y, _ = oracle.combine(eo, np.array([[0, 1, 2, 3]], np.int32), w[:, ::-1].copy())
    assert y[0, 0] == 0x3F81


def test_combine_uses_fused_multiply_add():
    # k0: 1 * -(1 + 2^-7);  k1: (1 + 2^-23) * (1 + 2^-7) = 1 + 2^-7 + 2^-23 + 2^-30.
    # fused: the sum is 2^-23 (1 + 2^-7) exactly -> BF16 0x3401.
    # separate multiply then add would drop 2^-30 -> 2^-23 -> 0x3400.
    a = 1.0 + 2.0 ** -7
    eo = np.array([[_bf16_of(-a)], [_bf16_of(a)]], np.uint16).repeat(128, axis=1)
    w = np.array([[1.0, 1.0 + 2.0 ** -23]], np.float32)
    y, _ = oracle.combine(eo, np.array([[0, 1]], np.int32), w)
    assert y[0, 0] == 0x3401


@pytest.mark.parametrize("name,tol_ulps", [("normal", None), ("bf16", 1)])
def test_identity_roundtrip(name, tol_ulps):
    w = make_workload(name, seed=0, num_tokens=96, hidden=512 if name == "normal" else 256)
    d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, w.num_experts, w.num_partitions,
                        quant=w.quant)
    eo = oracle.identity_expert(d["recv_x"], d["recv_scales"], quant=w.quant)
    y, st = oracle.combine(eo, d["row_of"], w.topk_weights)
    assert st == 0
    x = f32_from_bf16_bits(w.x).astype(np.float64)
    yf = f32_from_bf16_bits(y).astype(np.float64)
    if tol_ulps is not None:
        # BF16 path: no quantisation; weights sum to 1 within float32 rounding
        ulp = np.abs(x) * 2.0 ** -7 + 1e-38
        assert np.all(np.abs(yf - x) <= tol_ulps * ulp)
    else:
        # FP8: per element error <= 2^-4 |x| (+ subnormal step) + BF16 rounding
        s = np.repeat(oracle.quantize_rows(w.x)[1].astype(np.float64), 128, axis=1)
        bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * s) * 1.01 + np.abs(x) * 2.0 ** -7
        assert np.all(np.abs(yf - x) <= bound)


def test_identity_roundtrip_with_masks_scales_by_weight_sum():
    w = make_workload("skew", seed=0, num_tokens=64, hidden=256)
    d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 256, 8)
    eo = oracle.identity_expert(d["recv_x"], d["recv_scales"])
    y, _ = oracle.combine(eo, d["row_of"], w.topk_weights)
    wsum = np.where(w.topk_idx >= 0, w.topk_weights, 0).sum(axis=1, dtype=np.float64)
    x = f32_from_bf16_bits(w.x).astype(np.float64) * wsum[:, None]
    yf = f32_from_bf16_bits(y).astype(np.float64)
    xa = f32_from_bf16_bits(w.x).astype(np.float64)
    assert np.all(np.abs(yf - x) <= 2.0 ** -4 * np.abs(xa) * 1.01 + np.abs(x) * 2.0 ** -7 + 1e-6)


def test_ll_agrees_with_normal_layout():
    w = make_workload("ll", seed=0, hidden=256)
    cap = w.num_max_tokens
    d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 256, 8)
    ll = oracle.ll_dispatch(w.x, w.topk_idx, 256, cap)
    assert ll["status"] == 0
    assert np.array_equal(ll["recv_expert_count"], d["num_tokens_per_expert"])
    off = d["expert_offset"]
    for e in range(256):
        n = ll["recv_expert_count"][e]
        assert np.array_equal(ll["recv_x"][e, :n], d["recv_x"][off[e]:off[e] + n])
        assert np.array_equal(ll["recv_scales"][e, :n], d["recv_scales"][off[e]:off[e] + n])
        assert np.array_equal(ll["ll_src_of"][e, :n], d["src_of"][off[e]:off[e] + n])
        assert np.all(ll["recv_x"][e, n:] == 0xA5)  # padding untouched
    # ll_row_of = e * cap + (row - expert_offset[e])
    e_of = w.topk_idx
    want = e_of * cap + (d["row_of"] - off[e_of])
    assert np.array_equal(ll["ll_row_of"], want)
    # LL combine == normal combine, bit for bit
    eo_n = oracle.identity_expert(d["recv_x"], d["recv_scales"])
    eo_ll = np.zeros((256, cap, 256), np.uint16)
    for e in range(256):
        n = ll["recv_expert_count"][e]
        eo_ll[e, :n] = eo_n[off[e]:off[e] + n]
    y_n, _ = oracle.combine(eo_n, d["row_of"], w.topk_weights)
    y_ll, _ = oracle.ll_combine(eo_ll, ll["ll_row_of"], w.topk_weights)
    assert np.array_equal(y_n, y_ll)


def test_ll_capacity_overflow_is_reported_and_dropped():
    # every token names expert 2 twice (duplicates) -> 2*T rows for a capacity of T
    T, K, E = 6, 2, 4
    idx = np.full((T, K), 2, np.int64)
    x = random_bf16(np.random.default_rng(0), (T, 128))
    ll = oracle.ll_dispatch(x, idx, E, T)
    assert ll["status"] & oracle.CAPACITY
    assert ll["recv_expert_count"][2] == T
    assert np.array_equal(ll["ll_row_of"].reshape(-1)[:T], 2 * T + np.arange(T))
    assert np.all(ll["ll_row_of"].reshape(-1)[T:] == -1)


def test_empty_batch():
    idx = np.zeros((0, 8), np.int64)
    lay = oracle.layout(idx, 16, 4)
    assert lay["num_recv"][0] == 0 and np.all(lay["expert_offset"] == 0)
    assert np.all(lay["num_tokens_per_expert"] == 0)
    d = oracle.dispatch(np.zeros((0, 128), np.uint16), idx, np.zeros((0, 8), np.float32), 16, 4)
    assert d["recv_x"].shape == (0, 128)
