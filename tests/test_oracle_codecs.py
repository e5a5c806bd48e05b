"""Pins for the oracle's number formats: E4M3, BF16, the 1x128 block scale.

The DeepEP pages say dispatch is FP8 and combine is BF16 ("DeepSeek 开源周第二弹：
DeepEP", section "DeepEP 的常规内核和低延迟内核") but print no conversion example,
so the oracle's codecs are pinned against what the format definitions and
independent implementations fix:

* E4M3 decoding: torch's ``float8_e4m3fn`` dtype, all 256 codes, plus closed
  forms of the OCP FP8 definition (bias 7, largest finite 448, subnormal
  step 2^-9).
* E4M3 encoding: a brute-force nearest-value search over the 127 finite
  magnitudes (ties to the even code), on every code value, every midpoint and
  its neighbours one float32 ulp away, and a random sample; torch's cast on
  2M random values inside [-448, 448] (outside it torch returns NaN instead
  of saturating, so the two are not compared there).
* BF16 rounding: torch's float32 -> bfloat16 cast on random bit patterns.
* Power-of-two (UE8M0) scales: the scale is a power of two and the smallest
  one not below the plain scale; codes are torch's cast of the exact quotient.
"""
import numpy as np
import pytest
import torch

import oracle


def _f32_bits(v):
    return np.asarray(v, dtype=np.float32).view(np.uint32)


# ------------------------------------------------------------------- E4M3 --

def _e4m3_table():
    """The 127 non-negative finite E4M3 magnitudes with their codes, from the
    definition: code c = E<<3 | m; E == 0 -> m * 2^-9, else (1 + m/8) 2^(E-7)."""
    codes = np.arange(0x7F, dtype=np.int64)  # 0x00 .. 0x7E (0x7F is NaN)
    E = codes >> 3
    m = codes & 7
    val = np.where(E == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (E - 7))
    return codes, val


def _brute_e4m3(v):
    """Nearest finite E4M3 value (ties to the even code), |v| > 448 -> 448."""
    codes, table = _e4m3_table()
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    out = np.empty(v.shape, dtype=np.uint8)
    for lo in range(0, v.size, 1 << 15):
        aa = a[lo:lo + (1 << 15)]
        d = np.abs(aa[:, None] - table[None, :])
        dmin = d.min(axis=1, keepdims=True)
        cand = d == dmin
        # among the (at most two) nearest, prefer the even code
        even = cand & ((codes[None, :] & 1) == 0)
        pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
        c = codes[pick]
        c = np.where(aa > 448.0, 0x7E, c)
        out[lo:lo + (1 << 15)] = c
    sign = (_f32_bits(v.astype(np.float32)) >> 31).astype(np.uint8)
    return out | (sign << 7)


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = np.array([oracle.e4m3_to_f32(int(c)) for c in codes], dtype=np.float32)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    nan_ours, nan_ref = np.isnan(ours), np.isnan(ref)
    assert np.array_equal(nan_ours, nan_ref)
    assert set(np.nonzero(nan_ours)[0]) == {0x7F, 0xFF}
    assert np.array_equal(_f32_bits(ours[~nan_ours]), _f32_bits(ref[~nan_ref]))


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x80, -0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x38, 1.0), (0x3C, 1.5), (0x40, 2.0), (0x76, 224.0), (0x7E, 448.0), (0xFE, -448.0),
    (0x77, 240.0), (0x70, 128.0),
])
def test_e4m3_closed_forms(code, value):
    got = oracle.e4m3_to_f32(code)
    assert got == value and np.signbit(got) == np.signbit(value)
    assert oracle.e4m3_from_f32(value) == code


def test_e4m3_roundtrip_all_finite_codes():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_from_f32(oracle.e4m3_to_f32(c)) == c


def test_e4m3_midpoints_and_neighbours_vs_bruteforce():
    _, table = _e4m3_table()
    mids = (table[:-1] + table[1:]) / 2.0  # exact in float32 (<= 5 significant bits)
    pts = np.concatenate([table, mids, [448.0, 464.0, 479.9, 480.0, 1e4, 3.0e38]]).astype(np.float32)
    up = np.nextafter(pts, np.float32(np.inf))
    dn = np.nextafter(pts, np.float32(0))
    allp = np.concatenate([pts, up, dn])
    allp = np.concatenate([allp, -allp])
    ours = oracle.e4m3_from_f32_array(allp)
    assert np.array_equal(ours, _brute_e4m3(allp))
    # ties go to the even mantissa: 1.0625 lies halfway between 1.0 (0x38) and 1.125 (0x39)
    assert oracle.e4m3_from_f32(1.0625) == 0x38
    assert oracle.e4m3_from_f32(1.1875) == 0x3A  # between 0x39 and 0x3A -> even 0x3A
    assert oracle.e4m3_from_f32(2.0 ** -10) == 0x00  # half the smallest subnormal -> 0
    assert oracle.e4m3_from_f32(3 * 2.0 ** -10) == 0x02  # between 0x01 and 0x02 -> even


def test_e4m3_random_vs_bruteforce():
    rng = np.random.default_rng(7)
    mag = np.exp2(rng.uniform(-14, 9.2, size=120_000)).astype(np.float32)
    sgn = np.where(rng.random(mag.size) < 0.5, -1.0, 1.0).astype(np.float32)
    v = mag * sgn
    assert np.array_equal(oracle.e4m3_from_f32_array(v), _brute_e4m3(v))


def test_e4m3_saturates_and_keeps_sign():
    for v, c in [(448.0, 0x7E), (449.0, 0x7E), (463.9, 0x7E), (464.0, 0x7E), (1e9, 0x7E),
                 (float("inf"), 0x7E), (-500.0, 0xFE), (float("-inf"), 0xFE), (-0.0, 0x80),
                 (-1e-30, 0x80), (1e-30, 0x00)]:
        assert oracle.e4m3_from_f32(v) == c, (v, c)
    assert oracle.e4m3_from_f32(float("nan")) & 0x7F == 0x7F


def test_e4m3_matches_torch_cast_inside_range():
    rng = np.random.default_rng(11)
    a = np.concatenate([
        rng.uniform(-448, 448, 1_000_000),
        np.exp2(rng.uniform(-16, np.log2(448.0), 1_000_000)) * np.where(rng.random(1_000_000) < .5, -1, 1),
    ]).astype(np.float32)
    a = a[np.abs(a) <= 448.0]
    ref = torch.from_numpy(a).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_from_f32_array(a), ref)


# ------------------------------------------------------------------- BF16 --

def test_bf16_matches_torch_random_bits():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[~np.isnan(v)]
    ref = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_from_f32_array(v), ref)


def test_bf16_ties_to_even():
    # low half exactly 0x8000: round to the even upper half
    for hi in (0x3F80, 0x3F81, 0xBF80, 0xBF81, 0x7F7F):
        v = np.array([(hi << 16) | 0x8000], dtype=np.uint32).view(np.float32)[0]
        want = hi + (hi & 1)
        assert oracle.bf16_from_f32(float(v)) == want
    assert oracle.bf16_from_f32(1.0) == 0x3F80
    assert oracle.bf16_from_f32(-2.0) == 0xC000
    assert oracle.bf16_to_f32(0x3F80) == 1.0


# ---------------------------------------------------------------- scales --

def test_block_scale_closed_forms():
    f32 = np.float32
    assert oracle.block_scale(448.0) == 1.0
    assert oracle.block_scale(224.0) == 0.5
    assert oracle.block_scale(896.0) == 2.0
    floor = oracle.block_scale(0.0)
    # the amax floor 1e-4 applies at and below 1e-4
    assert floor == oracle.block_scale(1e-5) == oracle.block_scale(float(f32(1e-4)))
    assert abs(floor * 448.0 - 1e-4) <= 1e-4 * 2.0 ** -22
    assert oracle.block_scale(2e-4) > floor


def test_quantize_zero_block():
    x = np.zeros(256, np.uint16)
    q, s = oracle.quantize_row(x)
    assert np.all(q == 0)
    assert np.all(s == np.float32(oracle.block_scale(0.0)))


def test_quantize_amax_448_block_is_plain_cast():
    rng = np.random.default_rng(5)
    f = rng.uniform(-448, 448, 128).astype(np.float32)
    f[17] = 448.0
    x = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, s = oracle.quantize_row(x)
    assert s[0] == 1.0
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    ref = torch.from_numpy(xf.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def test_quantize_worked_block():
    # amax = 2 -> scale = 2/448; 1.0 / scale = 224 -> code 0x76; amax -> 448 -> 0x7E
    f = np.zeros(128, np.float32)
    f[0], f[1], f[2], f[3] = 2.0, 1.0, -0.5, -2.0
    x = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, s = oracle.quantize_row(x)
    assert s[0] == np.float32(2.0) / np.float32(448.0)
    assert list(q[:4]) == [0x7E, 0x76, 0xEE, 0xFE]
    assert np.all(q[4:] == 0)


def test_quantize_roundtrip_error_bound_and_block_independence():
    rng = np.random.default_rng(9)
    H = 1024
    f = rng.standard_normal(H).astype(np.float32)
    f[128:256] *= 100.0  # an outlier block
    f[512:640] *= 1e-6   # a block under the amax floor
    x = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    q, s = oracle.quantize_row(x)
    deq = np.array([oracle.e4m3_to_f32(int(c)) for c in q]) * np.repeat(s.astype(np.float64), 128)
    bound = np.maximum(2.0 ** -4 * np.abs(xf), 2.0 ** -10 * np.repeat(s.astype(np.float64), 128))
    assert np.all(np.abs(deq - xf) <= bound * (1 + 2.0 ** -20))
    # the largest magnitude of every block above the floor maps to +-448
    for b in range(H // 128):
        blk = np.abs(xf[b * 128:(b + 1) * 128])
        if blk.max() > 1e-4:
            assert (q[b * 128:(b + 1) * 128] & 0x7F).max() == 0x7E
    # changing one block leaves the others' codes and scales alone
    x2 = x.copy()
    x2[300] ^= 0x0100
    q2, s2 = oracle.quantize_row(x2)
    other = np.ones(H, bool)
    other[256:384] = False
    assert np.array_equal(q[other], q2[other])
    assert np.array_equal(np.delete(s, 2), np.delete(s2, 2))


# ------------------------------------------------------- power-of-two scales --

def test_pow2_scale_closed_forms_and_bracket():
    assert oracle.block_scale_pow2(448.0) == 1.0
    assert oracle.block_scale_pow2(449.0) == 2.0
    assert oracle.block_scale_pow2(224.0) == 0.5
    assert oracle.block_scale_pow2(0.0) == 2.0 ** -22  # 1e-4 / 448 = 2.23e-7 -> 2^-22
    rng = np.random.default_rng(12)
    for a in np.exp2(rng.uniform(-20, 20, 2000)).astype(np.float32):
        s = oracle.block_scale_pow2(float(a))
        r = oracle.block_scale(float(a))
        m, _ = np.frexp(s)
        assert m == 0.5                  # a power of two
        assert s >= r and s / 2 < r      # the smallest one not below the plain scale


def test_pow2_quantise_matches_torch_cast_of_exact_quotient():
    rng = np.random.default_rng(13)
    f = (rng.standard_normal(1024) * np.exp2(rng.uniform(-6, 6, 1024))).astype(np.float32)
    x = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, s = oracle.quantize_row(x, pow2=True)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    quot = (xf / np.repeat(s, 128)).astype(np.float32)  # division by a power of two: exact
    assert np.all(np.abs(quot) <= 448.0)
    ref = torch.from_numpy(quot).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def test_pow2_dispatch_rows_are_pow2_quantised_token_rows():
    from workloads import make_workload
    w = make_workload("normal", seed=3, num_tokens=40, hidden=256)
    d = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 256, 8, quant="fp8_pow2")
    d1 = oracle.dispatch(w.x, w.topk_idx, w.topk_weights, 256, 8, quant="fp8")
    R = int(d["num_recv"][0])
    assert R == int(d1["num_recv"][0]) and np.array_equal(d["src_of"], d1["src_of"])
    for r in range(R):
        t = int(d["src_of"][r]) // w.num_topk
        q, s = oracle.quantize_row(w.x[t], pow2=True)
        assert np.array_equal(d["recv_x"][r], q) and np.array_equal(d["recv_scales"][r], s)
    # the power-of-two scales never fall below the plain ones
    assert np.all(d["recv_scales"][:R] >= d1["recv_scales"][:R])
