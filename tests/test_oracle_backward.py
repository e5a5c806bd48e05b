"""Pins for the oracle's backward pair (dispatch backward, combine backward).

Checked against what the definitions fix: float64 sums of the gathered rows
with the fp32 rounding bound, exact single-slot cases, torch's float32 ->
bfloat16 cast for the scaled gradient rows, numpy's float64 dot products for
the topk_weights gradient (the products of two BF16 values are exact in
float32, so an exact float64 sum does not depend on the order), and the
adjoint identity <grad_y, combine(eo)> = sum over rows <grad_eo, eo> in exact
arithmetic.
"""
import numpy as np
import torch

import oracle
from workloads import f32_from_bf16_bits, make_custom, random_bf16


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _case(seed, T=29, K=4, E=12, P=3, H=256, mask=0.15):
    w = make_custom(T, H, K, E, P, seed=seed, mask_frac=mask)
    lay = oracle.layout(w.topk_idx, E, P)
    return w, lay


def test_dispatch_backward_single_slot_is_a_copy():
    rng = np.random.default_rng(0)
    g = random_bf16(rng, (7, 128))
    row_of = np.array([[3], [0], [6], [-1]], np.int32)
    gx, _, st = oracle.dispatch_backward(g, row_of)
    assert st == 0
    assert np.array_equal(gx[:3], g[[3, 0, 6]])
    assert np.all(gx[3] == 0)  # a token with no valid slot gets +0


def test_dispatch_backward_vs_float64_bound():
    for seed in range(3):
        w, lay = _case(seed)
        R = int(lay["num_recv"][0])
        rng = np.random.default_rng(seed + 10)
        g = random_bf16(rng, (R, 256))
        gx, _, st = oracle.dispatch_backward(g, lay["row_of"])
        assert st == 0
        gf = f32_from_bf16_bits(g).astype(np.float64)
        exact = np.zeros((w.num_tokens, 256))
        mag = np.zeros_like(exact)
        for t in range(w.num_tokens):
            for r in lay["row_of"][t]:
                if r >= 0:
                    exact[t] += gf[r]
                    mag[t] += np.abs(gf[r])
        got = f32_from_bf16_bits(gx).astype(np.float64)
        bound = 4 * 2.0 ** -24 * mag + np.abs(exact) * 2.0 ** -8
        assert np.all(np.abs(got - exact) <= bound * 1.01 + 1e-30)


def test_dispatch_backward_weight_gradient_is_a_gather():
    w, lay = _case(5)
    R = int(lay["num_recv"][0])
    grw = np.random.default_rng(1).standard_normal(R).astype(np.float32)
    _, gw, _ = oracle.dispatch_backward(np.zeros((R, 256), np.uint16), lay["row_of"], grw)
    for t in range(w.num_tokens):
        for k in range(w.num_topk):
            r = lay["row_of"][t, k]
            assert gw[t, k] == (grw[r] if r >= 0 else 0.0)


def test_combine_backward_rows_weights_and_untouched():
    w, lay = _case(7)
    R = int(lay["num_recv"][0])
    rng = np.random.default_rng(3)
    gy = random_bf16(rng, (w.num_tokens, 256))
    eo = random_bf16(rng, (R + 5, 256))  # 5 rows no slot points at
    geo, gw, st = oracle.combine_backward(gy, eo, lay["row_of"], w.topk_weights)
    assert st == 0
    gyf = f32_from_bf16_bits(gy)
    eof = f32_from_bf16_bits(eo).astype(np.float64)
    seen = set()
    for t in range(w.num_tokens):
        for k in range(w.num_topk):
            r = lay["row_of"][t, k]
            if r < 0:
                assert gw[t, k] == 0.0
                continue
            seen.add(int(r))
            want_row = _bf16(np.float32(w.topk_weights[t, k]) * gyf[t])
            assert np.array_equal(geo[r], want_row)
            want_w = np.float32(np.dot(gyf[t].astype(np.float64), eof[r]))
            assert gw[t, k] == want_w
    untouched = sorted(set(range(R + 5)) - seen)
    assert len(untouched) >= 5 and np.all(geo[untouched] == 0xA5A5)


def test_combine_backward_adjoint_identity():
    # exact arithmetic: <grad_y, sum_k w e_k> = sum_rows <w g, e_row>; the oracle's
    # rows are w*g rounded to BF16, so compare within that rounding
    w, lay = _case(11, T=17, K=3, E=9, P=3, H=128, mask=0.0)
    R = int(lay["num_recv"][0])
    rng = np.random.default_rng(4)
    gy = random_bf16(rng, (w.num_tokens, 128))
    eo = random_bf16(rng, (R, 128))
    geo, gw, _ = oracle.combine_backward(gy, eo, lay["row_of"], w.topk_weights)
    gyf = f32_from_bf16_bits(gy).astype(np.float64)
    eof = f32_from_bf16_bits(eo).astype(np.float64)
    lhs = 0.0
    for t in range(w.num_tokens):
        y = np.zeros(128)
        for k in range(3):
            y += float(w.topk_weights[t, k]) * eof[lay["row_of"][t, k]]
        lhs += float(np.dot(gyf[t], y))
    rhs = float(np.sum(f32_from_bf16_bits(geo).astype(np.float64) * eof))
    scale = float(np.sum(np.abs(f32_from_bf16_bits(geo).astype(np.float64) * eof)))
    assert abs(lhs - rhs) <= 2.0 ** -8 * scale
    # and the weight gradients sum to the same inner product, weighted
    lhs_w = float(np.sum(gw.astype(np.float64) * w.topk_weights.astype(np.float64)))
    assert abs(lhs_w - lhs) <= 1e-5 * scale
