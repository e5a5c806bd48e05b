// ep_quant.cuh -- the FP8 quantiser shared by the normal and low-latency dispatch kernels.
//
// Per 128-channel block of a BF16 row: amax = max |x|, s = max(amax, 1e-4) / 448
// (one IEEE fp32 division), q = e4m3(x / s) with the fp32 quotient rounded to
// nearest-even and saturated to +-448 (cvt.rn.satfinite).  The pages fix only
// "FP8 dispatch" ("DeepSeek 开源周第二弹：DeepEP", section "DeepEP 的常规内核和低延迟
// 内核"); E4M3 with 1x128 fp32 scales is this library's reading.
//
// The per-element quotient x / s is formed with Markstein's correction step
// (P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Develop. 34(1), 1990; also Muller et al., "Handbook of
// Floating-Point Arithmetic", the chapter on division): with y = RN(1/s) (one
// correctly rounded reciprocal per block) and q0 = RN(x * y), the residual
// r = x - q0 * s is exact in one fused multiply-add and RN(q0 + r * y) is the
// correctly rounded quotient RN(x / s) whenever nothing underflows.  Here
// |x / s| <= 448 (no overflow) and s >= 1e-4 / 448 is normal; a quotient small
// enough for anything to underflow (below 2^-126) is far below half the smallest
// E4M3 subnormal (2^-10), so its E4M3 code is a signed zero either way, and the
// sign is restored with copysign (RN(x / s) always has the sign of x).  The codes
// are therefore those of the IEEE division, at 4 instructions per element.
#pragma once

#include "ep_device.cuh"

namespace ep {

// Quantise one BF16 row held in shared memory.  A warp takes two 128-channel
// blocks at a time: lanes 0-15 the even block, lanes 16-31 the odd one, 8
// channels (16 bytes) per lane; the block amax is a 16-lane xor-shuffle max.
//
// pow2: round each scale up to the next power of two (for consumers that take
// scales as an 8-bit exponent); x / s is then an exact exponent shift.
__device__ __forceinline__ float quotient_rn(float x, float s, float y) {
    const float q0 = __fmul_rn(x, y);
    const float r = __fmaf_rn(-q0, s, x);
    return copysignf(__fmaf_rn(r, y, q0), x);
}

// s = RN(max(amax, 1e-4) / 448), by the same correction step with the constant
// y = RN(1 / 448) (a positive normal quotient: no underflow, no sign question).
__device__ __forceinline__ float block_scale(float amax) {
    constexpr float kInv448 = 1.0f / 448.0f;  // RN(1/448), folded at compile time
    const float a = fmaxf(amax, 1e-4f);
    const float q0 = __fmul_rn(a, kInv448);
    return __fmaf_rn(__fmaf_rn(-q0, 448.0f, a), kInv448, q0);
}

// One 128-channel block held by 16 lanes (8 channels each): scale and codes.
__device__ __forceinline__ void quantize_block8(uint4 v, bool pow2, float* s_out, uint2* q_out) {
    float f[8];
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 8));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    float s = block_scale(amax);
    if (pow2) {
        const uint32_t b = __float_as_uint(s);  // s is normal and positive
        if (b & 0x007FFFFFu) s = __uint_as_float((b & 0x7F800000u) + 0x00800000u);
    }
    const float y = __frcp_rn(s);
    float d[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) d[j] = quotient_rn(f[j], s, y);
    q_out->x = e4m3x2(d[0], d[1]) | (e4m3x2(d[2], d[3]) << 16);
    q_out->y = e4m3x2(d[4], d[5]) | (e4m3x2(d[6], d[7]) << 16);
    *s_out = s;
}

// Quantise one BF16 row held in shared memory.  A warp takes two 128-channel
// blocks at a time: lanes 0-15 the even block, lanes 16-31 the odd one, 8
// channels (16 bytes) per lane; the block amax is a 16-lane xor-shuffle max.
// Two such block pairs are worked on together where the warp has them, so that
// their latency chains (shared-memory load, shuffles, reciprocal) overlap.
//
// pow2: round each scale up to the next power of two (for consumers that take
// scales as an 8-bit exponent); x / s is then an exact exponent shift.
__device__ __forceinline__ void quantize_row_fp8(const uint8_t* __restrict__ in,
                                             uint8_t* __restrict__ out_q,
                                             float* __restrict__ out_s, int nb, int warp,
                                             int nwarps, int lane, bool pow2 = false) {
    const int half = lane >> 4, l16 = lane & 15;
    const uint4* src = reinterpret_cast<const uint4*>(in);
    uint2* dst = reinterpret_cast<uint2*>(out_q);
    int bp = warp;
    for (; 2 * (bp + nwarps) < nb; bp += 2 * nwarps) {  // two pairs: bp and bp + nwarps
        const int b0 = 2 * bp + half, b1 = 2 * (bp + nwarps) + half;
        const bool act1 = b1 < nb;  // b0 < nb holds: 2 * bp + 1 < 2 * (bp + nwarps) < nb
        const uint4 v0 = src[b0 * 16 + l16];
        const uint4 v1 = act1 ? src[b1 * 16 + l16] : make_uint4(0u, 0u, 0u, 0u);
        float s0, s1;
        uint2 q0, q1;
        quantize_block8(v0, pow2, &s0, &q0);
        quantize_block8(v1, pow2, &s1, &q1);
        dst[b0 * 16 + l16] = q0;
        if (l16 == 0) out_s[b0] = s0;
        if (act1) {
            dst[b1 * 16 + l16] = q1;
            if (l16 == 0) out_s[b1] = s1;
        }
    }
    for (; 2 * bp < nb; bp += nwarps) {
        const int b = 2 * bp + half;
        const bool act = b < nb;
        const uint4 v = act ? src[b * 16 + l16] : make_uint4(0u, 0u, 0u, 0u);
        float s;
        uint2 q;
        quantize_block8(v, pow2, &s, &q);
        if (act) {
            dst[b * 16 + l16] = q;
            if (l16 == 0) out_s[b] = s;
        }
    }
}

}  // namespace ep
