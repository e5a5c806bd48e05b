"""GPU parity of the redundant-expert calls against the oracle: byte-exact weight
prefetch and bit-exact fp32 gradient reduce (same ascending slot order), on random
primary maps, the stress workload's 288-slot map, malformed entries and the
Buffer methods."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
from workloads import make_workload  # noqa: E402

from gpu_path import new_workspace  # noqa: E402


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import combine_get_dispatch_05_b200 as m
    return m


def _map(rng, S, groups):
    prim = np.sort(rng.choice(S, groups, replace=False)).astype(np.int32)
    po = rng.choice(prim, S).astype(np.int32)
    po[prim] = prim
    return po


MAPS = [("random-37", 37, 11, 4096), ("random-300", 300, 250, 65536 + 48),
        ("one-slot", 1, 1, 16), ("all-replicas-of-one", 20, 1, 1024)]


@pytest.mark.parametrize("name,S,groups,nbytes", MAPS, ids=[m[0] for m in MAPS])
def test_lb_prefetch_parity(ep, name, S, groups, nbytes):
    rng = np.random.default_rng(S)
    po = _map(rng, S, groups)
    w = rng.integers(0, 256, (S, nbytes), dtype=np.uint8)
    want, st = oracle.lb_prefetch_weights(w, po)
    dw = torch.from_numpy(w).cuda()
    ws = new_workspace(ep, 1, 1, 1)
    ep.ep_lb_prefetch_weights(torch.from_numpy(po).cuda(), dw, ws)
    assert np.array_equal(dw.cpu().numpy(), want)
    assert ep.ep_read_status(ws) == st == 0


@pytest.mark.parametrize("name,S,groups,n", [("random-37", 37, 11, 1000), ("random-300", 300, 250, 4100),
                                             ("big-group", 40, 2, 2052), ("one-slot", 1, 1, 8)])
def test_lb_reduce_parity(ep, name, S, groups, n):
    rng = np.random.default_rng(S + n)
    po = _map(rng, S, groups)
    g = (rng.standard_normal((S, n)) * np.exp2(rng.integers(-20, 20, (S, 1)))).astype(np.float32)
    g[0, :3] = [-0.0, np.float32(1e-45), 3e38]
    want, st = oracle.lb_reduce_grads(g, po)
    dg = torch.from_numpy(g).cuda()
    ws = new_workspace(ep, 1, 1, 1)
    ep.ep_lb_reduce_grads(torch.from_numpy(po).cuda(), dg, ws)
    assert np.array_equal(dg.cpu().numpy().view(np.uint32), want.view(np.uint32))
    assert ep.ep_read_status(ws) == st == 0


def test_lb_stress_map_and_buffer_methods(ep):
    w = make_workload("stress", seed=0, num_tokens=64, hidden=128)
    po = w.meta["primary_of"]
    S = po.size
    rng = np.random.default_rng(5)
    wt = rng.integers(0, 256, (S, 4096), dtype=np.uint8)
    g = rng.standard_normal((S, 512)).astype(np.float32)
    buf = ep.Buffer(num_experts=S, num_partitions=8, max_tokens=64)
    dpo = torch.from_numpy(po).cuda()
    dw, dg = torch.from_numpy(wt).cuda(), torch.from_numpy(g).cuda()
    buf.lb_prefetch_weights(dpo, dw).synchronize()
    buf.lb_reduce_grads(dpo, dg).synchronize()
    assert np.array_equal(dw.cpu().numpy(), oracle.lb_prefetch_weights(wt, po)[0])
    assert np.array_equal(dg.cpu().numpy().view(np.uint32),
                          oracle.lb_reduce_grads(g, po)[0].view(np.uint32))
    assert buf.read_status() == 0


def test_lb_malformed_entries_are_skipped_and_reported(ep):
    po = np.array([0, 0, 7, 1, 4], np.int32)  # slot 2 out of range, slot 3 names a replica
    w = np.arange(5 * 32, dtype=np.uint8).reshape(5, 32)
    g = np.ones((5, 4), np.float32)
    ws = new_workspace(ep, 1, 1, 1)
    dpo = torch.from_numpy(po).cuda()
    dw, dg = torch.from_numpy(w).cuda(), torch.from_numpy(g).cuda()
    ep.ep_lb_prefetch_weights(dpo, dw, ws)
    assert ep.ep_read_status(ws) == ep.EP_DEV_INDEX_RANGE
    ep.ep_lb_reduce_grads(dpo, dg, ws)
    assert ep.ep_read_status(ws) == ep.EP_DEV_INDEX_RANGE
    assert np.array_equal(dw.cpu().numpy(), oracle.lb_prefetch_weights(w, po)[0])
    assert np.array_equal(dg.cpu().numpy(), oracle.lb_reduce_grads(g, po)[0])
