"""GPU parity for the backward pair against the oracle, bit for bit.

dispatch backward: grad_x (fp32 sum of the token's row gradients in k order,
BF16 out) and the weight-gradient gather; combine backward: the scaled
gradient rows (fp32 multiply, BF16 out; rows no slot names untouched) and the
fp64 dot products of the weight gradient.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
from workloads import make_custom, make_workload, random_bf16  # noqa: E402

from gpu_path import bf16_to_u16, dev_u16_as_bf16, gpu_layout  # noqa: E402


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import combine_get_dispatch_05_b200 as m
    return m


CASES = [
    ("normal-300", lambda: make_workload("normal", seed=1, num_tokens=300, hidden=512)),
    ("skew-700", lambda: make_workload("skew", seed=2, num_tokens=700, hidden=256)),
    ("bf16-600", lambda: make_workload("bf16", seed=4, num_tokens=600, hidden=136)),
    ("k32-dups", lambda: make_custom(70, 128, 32, 48, 6, seed=8, duplicates=True)),
    ("e1", lambda: make_custom(33, 128, 2, 1, 1, seed=9, duplicates=True)),
    ("masked", lambda: make_custom(513, 640, 6, 64, 16, seed=10, mask_frac=0.3)),
    ("t1", lambda: make_custom(1, 128, 8, 256, 8, seed=6)),
]


@pytest.mark.parametrize("name,mk", CASES, ids=[c[0] for c in CASES])
def test_dispatch_backward_parity(ep, name, mk):
    w = mk()
    lay, ws = gpu_layout(ep, w.topk_idx, w.num_experts, w.num_partitions)
    want_lay = oracle.layout(w.topk_idx, w.num_experts, w.num_partitions)
    R = int(want_lay["num_recv"][0])
    rng = np.random.default_rng(5)
    g = random_bf16(rng, (R, w.hidden), scale=2.0)
    grw = rng.standard_normal(max(R, 1)).astype(np.float32)
    gx = torch.empty((w.num_tokens, w.hidden), dtype=torch.bfloat16, device="cuda")
    gw = torch.empty((w.num_tokens, w.num_topk), dtype=torch.float32, device="cuda")
    g_d = dev_u16_as_bf16(g) if R else torch.empty((0, w.hidden), dtype=torch.bfloat16,
                                                   device="cuda")
    ep.ep_dispatch_backward(g_d, lay, gx, ws, torch.from_numpy(grw).cuda(), gw)
    torch.cuda.synchronize()
    gx_ref, gw_ref, st = oracle.dispatch_backward(g, want_lay["row_of"], grw[:max(R, 1)])
    assert st == 0
    assert np.array_equal(bf16_to_u16(gx), gx_ref)
    assert np.array_equal(gw.cpu().numpy().view(np.uint32), gw_ref.view(np.uint32))
    assert ep.ep_read_status(ws) == 0


@pytest.mark.parametrize("name,mk", CASES, ids=[c[0] for c in CASES])
def test_combine_backward_parity(ep, name, mk):
    w = mk()
    lay, ws = gpu_layout(ep, w.topk_idx, w.num_experts, w.num_partitions)
    want_lay = oracle.layout(w.topk_idx, w.num_experts, w.num_partitions)
    R = int(want_lay["num_recv"][0])
    rng = np.random.default_rng(6)
    extra = 3  # rows no slot names: must stay untouched
    gy = random_bf16(rng, (w.num_tokens, w.hidden))
    eo = random_bf16(rng, (R + extra, w.hidden), scale=4.0)
    geo = torch.full(((R + extra) * w.hidden,), 0xA5A5 - 65536, dtype=torch.int16,
                     device="cuda").view(torch.bfloat16).view(R + extra, w.hidden)
    gw = torch.empty((w.num_tokens, w.num_topk), dtype=torch.float32, device="cuda")
    ep.ep_combine_backward(dev_u16_as_bf16(gy), dev_u16_as_bf16(eo), lay,
                           torch.from_numpy(w.topk_weights).cuda(), geo, gw, ws)
    torch.cuda.synchronize()
    geo_ref, gw_ref, st = oracle.combine_backward(gy, eo, want_lay["row_of"], w.topk_weights)
    assert st == 0
    assert np.array_equal(bf16_to_u16(geo), geo_ref)
    assert np.array_equal(gw.cpu().numpy().view(np.uint32), gw_ref.view(np.uint32))
    assert ep.ep_read_status(ws) == 0


def test_backward_full_size_sampled(ep):
    w = make_workload("normal", seed=3)
    T, H, K = w.num_tokens, w.hidden, w.num_topk
    lay, ws = gpu_layout(ep, w.topk_idx, 256, 8)
    want_lay = oracle.layout(w.topk_idx, 256, 8)
    R = int(want_lay["num_recv"][0])
    g_rows = torch.randn((R, H), device="cuda").to(torch.bfloat16)
    gy = torch.randn((T, H), device="cuda").to(torch.bfloat16)
    eo = torch.randn((R, H), device="cuda").to(torch.bfloat16)
    wts = torch.from_numpy(w.topk_weights).cuda()
    gx = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    geo = torch.empty_like(eo)
    gw = torch.empty((T, K), dtype=torch.float32, device="cuda")
    ep.ep_dispatch_backward(g_rows, lay, gx, ws)
    ep.ep_combine_backward(gy, eo, lay, wts, geo, gw, ws)
    torch.cuda.synchronize()
    assert ep.ep_read_status(ws) == 0
    rng = np.random.default_rng(9)
    sample = rng.choice(T, 24, replace=False)
    ro = want_lay["row_of"]
    for t in sample:
        rows = ro[t]
        rr = torch.from_numpy(rows.astype(np.int64)).cuda()
        # dispatch backward: the token's K row gradients, summed
        g_t = bf16_to_u16(g_rows[rr])
        ref, _, _ = oracle.dispatch_backward(g_t, np.arange(K, dtype=np.int32)[None, :])
        assert np.array_equal(bf16_to_u16(gx[t:t + 1]), ref), t
        # combine backward: this token's rows and weight gradients
        geo_ref, gw_ref, _ = oracle.combine_backward(
            bf16_to_u16(gy[t:t + 1]), bf16_to_u16(eo[rr]), np.arange(K, dtype=np.int32)[None, :],
            w.topk_weights[t:t + 1])
        assert np.array_equal(bf16_to_u16(geo[rr]), geo_ref), t
        assert np.array_equal(gw[t].cpu().numpy().view(np.uint32), gw_ref[0].view(np.uint32)), t
