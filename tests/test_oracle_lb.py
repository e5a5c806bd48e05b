"""Pins for the oracle's redundant-expert calls (weight prefetch, gradient reduce).

The pages ("deepseek-ai/DeepEP", sections "主要特性" and "典型工作流程", step 5)
name lb_prefetch_weights / lb_reduce_grads and say what they are for; nothing
numeric.  Pinned by what the reading fixes: after the prefetch every slot holds
its primary's bytes and primaries are untouched (and a second prefetch changes
nothing); the reduce gives exact group sums on integer-valued gradients (a
closed form), leaves singleton groups bit for bit, sums in ascending slot order
(a case where fp32 order changes the result), and leaves every slot of a group
equal; malformed maps are reported and skipped.
"""
import numpy as np

import oracle
from workloads import make_workload


def _map(rng, S, groups):
    """A random primary map: `groups` primaries, every other slot a replica."""
    prim = np.sort(rng.choice(S, groups, replace=False)).astype(np.int32)
    po = np.empty(S, np.int32)
    po[:] = rng.choice(prim, S)
    po[prim] = prim
    return po


def test_prefetch_copies_primary_blob_and_is_idempotent():
    rng = np.random.default_rng(0)
    S, nb = 37, 96
    po = _map(rng, S, 11)
    w = rng.integers(0, 256, (S, nb), dtype=np.uint8)
    out, st = oracle.lb_prefetch_weights(w, po)
    assert st == 0
    for s in range(S):
        assert np.array_equal(out[s], w[po[s]])  # every slot holds its primary's bytes
    prim = np.flatnonzero(po == np.arange(S))
    assert np.array_equal(out[prim], w[prim])  # primaries untouched
    again, _ = oracle.lb_prefetch_weights(out, po)
    assert np.array_equal(again, out)


def test_reduce_exact_on_integer_gradients():
    rng = np.random.default_rng(1)
    S, n = 29, 300
    po = _map(rng, S, 7)
    g = rng.integers(-1000, 1000, (S, n)).astype(np.float32)
    out, st = oracle.lb_reduce_grads(g, po)
    assert st == 0
    for q in np.unique(po):
        members = np.flatnonzero(po == q)
        want = g[members].astype(np.float64).sum(axis=0)  # exact: small integers
        for s in members:
            assert np.array_equal(out[s].astype(np.float64), want)


def test_reduce_singletons_unchanged_and_groups_equal():
    rng = np.random.default_rng(2)
    S, n = 16, 64
    po = np.arange(S, dtype=np.int32)
    po[[3, 9, 12]] = [1, 1, 5]
    g = rng.standard_normal((S, n)).astype(np.float32)
    g[0, :4] = [-0.0, 0.0, np.float32(1e-45), -3.5]
    out, _ = oracle.lb_reduce_grads(g, po)
    singles = [s for s in range(S) if (po == po[s]).sum() == 1]
    assert np.array_equal(out[singles].view(np.uint32), g[singles].view(np.uint32))
    assert np.array_equal(out[1], out[3]) and np.array_equal(out[1], out[9])
    assert np.array_equal(out[5], out[12])


def test_reduce_sums_in_ascending_slot_order():
    # (1e8 + 1) - 1e8 = 0 in binary32, while 1e8 - 1e8 + 1 = 1: the result fixes the order
    g = np.array([[1e8], [1.0], [-1e8], [7.0]], np.float32)
    po = np.array([0, 0, 0, 3], np.int32)
    out, _ = oracle.lb_reduce_grads(g, po)
    assert out[0, 0] == 0.0 and out[1, 0] == 0.0 and out[2, 0] == 0.0 and out[3, 0] == 7.0
    po2 = np.array([2, 2, 2, 3], np.int32)  # the same group under another primary: same order
    out2, _ = oracle.lb_reduce_grads(g, po2)
    assert np.array_equal(out2, out)


def test_malformed_maps_are_reported_and_skipped():
    w = np.arange(4 * 16, dtype=np.uint8).reshape(4, 16)
    po = np.array([0, 0, 7, 1], np.int32)  # slot 2 out of range, slot 3 names a replica
    out, st = oracle.lb_prefetch_weights(w, po)
    assert st == oracle.INDEX_RANGE
    assert np.array_equal(out[1], w[0]) and np.array_equal(out[2:], w[2:])
    g = np.ones((4, 3), np.float32)
    gout, st = oracle.lb_reduce_grads(g, po)
    assert st == oracle.INDEX_RANGE
    assert np.all(gout[0] == 2.0) and np.all(gout[1] == 2.0) and np.all(gout[2:] == 1.0)


def test_stress_workload_replica_map():
    w = make_workload("stress", seed=0, num_tokens=64, hidden=128)
    po = w.meta["primary_of"]
    S = w.num_experts
    assert po.shape == (S,) and S == 288
    prim = po == np.arange(S)
    assert prim.sum() == 256 and (~prim).sum() == 32
    assert np.all(prim[po])  # every replica names a primary
    # replica slots are the last 4 of each partition's 36
    assert np.array_equal(np.flatnonzero(~prim) % 36 >= 32, np.ones(32, bool))
