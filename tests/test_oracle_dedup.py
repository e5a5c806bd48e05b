"""Pins for the oracle's deduplicated (one row per token and partition) dispatch.

Brute force on the layout and the per-row expert lists (Python dicts), the
payload against the oracle's own row quantiser (one call per token), the
partition-local identity experts followed by the combine against x times the
token's weight sum within FP8 + BF16 error, and the row count: with top-4-group
routing a token reaches at most 4 of the 8 partitions, so the deduplicated
dispatch writes at most half the rows of the per-expert dispatch.
"""
import numpy as np

import oracle
from workloads import f32_from_bf16_bits, make_custom, make_workload, random_bf16


def _brute(idx, E, P):
    T, K = idx.shape
    epp = E // P
    parts = [sorted({int(e) // epp for e in idx[t] if 0 <= e < E}) for t in range(T)]
    rows = {}
    r = 0
    for p in range(P):
        for t in range(T):
            if p in parts[t]:
                rows[(t, p)] = r
                r += 1
    return rows, r


def test_dedup_layout_and_metadata_bruteforce():
    for seed, (T, K, E, P) in enumerate([(37, 4, 12, 3), (64, 8, 256, 8), (20, 3, 4, 4),
                                         (11, 6, 6, 1)]):
        w = make_custom(T, 128, K, E, P, seed=seed, mask_frac=0.1, duplicates=(seed % 2 == 1))
        d = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, E, P)
        rows, R = _brute(w.topk_idx, E, P)
        assert d["num_rows"][0] == R and d["status"] == 0
        epp = E // P
        for t in range(T):
            for p in range(P):
                want = rows.get((t, p), -1)
                assert d["prow_of"][t, p] == want
                if want < 0:
                    continue
                assert d["src_tok"][want] == t
                for k in range(K):
                    e = int(w.topk_idx[t, k])
                    inside = e >= 0 and e // epp == p
                    assert d["recv_topk_idx"][want, k] == (e - p * epp if inside else -1)
                    assert d["recv_topk_weights"][want, k] == (w.topk_weights[t, k] if inside
                                                               else 0.0)
        assert np.array_equal(d["part_offset"], np.concatenate([[0], np.cumsum(d["part_count"])]))


def test_dedup_payload_is_the_quantised_token_row():
    w = make_workload("normal", seed=2, num_tokens=50, hidden=256)
    d = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, 256, 8)
    for r, t in enumerate(d["src_tok"]):
        q, s = oracle.quantize_row(w.x[t])
        assert np.array_equal(d["recv_x"][r], q)
        assert np.array_equal(d["recv_scales"][r], s)


def test_dedup_halves_rows_under_group_limited_routing():
    w = make_workload("normal", seed=0, hidden=128)
    d = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, 256, 8)
    lay = oracle.layout(w.topk_idx, 256, 8)
    assert d["num_rows"][0] <= 4 * w.num_tokens
    assert d["num_rows"][0] * 2 <= lay["num_recv"][0]
    # partition row counts are the layout's distinct-token counts
    assert np.array_equal(d["part_count"], lay["num_tokens_per_partition"])


def test_dedup_identity_round_trip():
    w = make_workload("skew", seed=1, num_tokens=80, hidden=512)
    d = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, 256, 8)
    out = oracle.partition_identity(d["recv_x"], d["recv_scales"], d["recv_topk_idx"],
                                    d["recv_topk_weights"])
    y, st = oracle.combine_dedup(out, d["prow_of"])
    assert st == 0
    xa = f32_from_bf16_bits(w.x).astype(np.float64)
    wsum = np.where(w.topk_idx >= 0, w.topk_weights, 0).sum(axis=1, dtype=np.float64)
    want = xa * wsum[:, None]
    got = f32_from_bf16_bits(y).astype(np.float64)
    s = np.repeat(oracle.quantize_rows(w.x)[1].astype(np.float64), 128, axis=1)
    # FP8 (2^-4 relative, 2^-10 * scale in the subnormal range), BF16 rounding of
    # each partition row and of y
    fp8 = np.maximum(2.0 ** -4 * np.abs(xa), 2.0 ** -10 * s) * 1.01
    assert np.all(np.abs(got - want) <= fp8 + 3 * 2.0 ** -8 * (np.abs(xa) + fp8) + 1e-12)


def test_dedup_combine_single_partition_is_a_copy():
    part = random_bf16(np.random.default_rng(0), (5, 128))
    prow = np.array([[2], [0], [-1]], np.int32)
    y, _ = oracle.combine_dedup(part, prow)
    assert np.array_equal(y[:2], part[[2, 0]])
    assert np.all(y[2] == 0)


def test_dedup_bf16_payload_is_bit_copy():
    w = make_custom(33, 136, 5, 10, 5, seed=4, quant="none")
    d = oracle.dispatch_dedup(w.x, w.topk_idx, w.topk_weights, 10, 5, quant="none")
    assert np.array_equal(d["recv_x"], w.x[d["src_tok"]])
