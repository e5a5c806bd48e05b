"""The seeded workloads against the settings the pages print (tests/golden)
and against the properties each workload promises."""
import json
import os

import numpy as np

import oracle
from workloads import f32_from_bf16_bits, make_workload

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_settings.json")))


def test_normal_matches_pages_setting():
    g = GOLDEN["normal"]
    w = make_workload("normal", seed=0, hidden=128)
    assert (w.num_tokens, w.num_topk, w.quant) == (g["num_tokens"], g["num_topk"], "fp8")
    assert make_workload("normal", seed=0, num_tokens=4).hidden == g["hidden"]
    # group-limited: each token's experts fall in at most top-4 of the 8 groups
    groups = w.topk_idx // 32
    assert max(len(set(r)) for r in groups.tolist()) <= g["topk_groups"]
    assert np.all(np.array([len(set(r)) for r in w.topk_idx.tolist()]) == 8)
    assert np.allclose(w.topk_weights.sum(axis=1), 1.0, atol=1e-6)


def test_low_latency_matches_pages_setting_and_buffer_size():
    g = GOLDEN["low_latency"]
    w = make_workload("ll", seed=0, hidden=256)
    assert (w.num_tokens, w.num_topk) == (g["num_tokens"], g["num_topk"])
    assert make_workload("ll", seed=0, num_tokens=2).hidden == g["hidden"]
    # the padded receive tensor holds num_max_tokens * hidden * num_experts FP8 elements
    ll = oracle.ll_dispatch(w.x, w.topk_idx, w.num_experts, w.num_max_tokens)
    assert ll["recv_x"].size == w.num_max_tokens * w.hidden * w.num_experts
    assert ll["recv_x"].dtype.itemsize == 1


def test_skew_is_skewed_and_masked():
    w = make_workload("skew", seed=0, hidden=128)
    flat = w.topk_idx.reshape(-1)
    assert (flat == -1).sum() == round(0.05 * w.num_tokens * w.num_topk)
    cnt = np.bincount(flat[flat >= 0], minlength=256)
    assert cnt.max() > 10 * cnt.mean()
    for r in w.topk_idx.tolist():
        v = [e for e in r if e >= 0]
        assert len(v) == len(set(v))


def test_bf16_outliers():
    w = make_workload("bf16", seed=0, num_tokens=1000, hidden=64)
    assert w.quant == "none" and (w.num_topk, w.num_experts, w.num_partitions) == (6, 64, 16)
    rows = w.meta["outlier_rows"]
    assert len(rows) == 10
    mags = np.abs(f32_from_bf16_bits(w.x)).max(axis=1)
    assert mags[rows].min() > 20 * np.median(mags)


def test_stress_replica_slots():
    w = make_workload("stress", seed=0, num_tokens=2048, hidden=128)
    assert (w.num_experts, w.num_partitions) == (288, 8)
    idx = w.topk_idx
    assert idx.min() >= 0 and idx.max() < 288
    for r in idx.tolist():
        assert len(set(r)) == 8
    slot_in_part = idx % 36
    # replica slots (32..35 of each partition) only for odd tokens of hot experts
    rep = slot_in_part >= 32
    assert rep[0::2].sum() == 0 and rep[1::2].sum() > 0
    hot = set(w.meta["hottest"].tolist())
    logical = w.meta["logical_idx"]
    assert set(logical[rep].tolist()) <= hot


def test_generators_are_seeded():
    a = make_workload("normal", seed=3, num_tokens=64, hidden=128)
    b = make_workload("normal", seed=3, num_tokens=64, hidden=128)
    c = make_workload("normal", seed=4, num_tokens=64, hidden=128)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.topk_idx, b.topk_idx)
    assert not np.array_equal(a.topk_idx, c.topk_idx)
