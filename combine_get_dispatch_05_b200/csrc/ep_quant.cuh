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

__device__ __forceinline__ void quantize_row_fp8(const uint8_t* __restrict__ in,
                                             uint8_t* __restrict__ out_q,
                                             float* __restrict__ out_s, int nb, int warp,
                                             int nwarps, int lane, bool pow2 = false) {
    const int half = lane >> 4, l16 = lane & 15;
    for (int bp = warp; 2 * bp < nb; bp += nwarps) {
        const int b = 2 * bp + half;
        const bool act = b < nb;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (act) v = reinterpret_cast<const uint4*>(in)[b * 16 + l16];
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
        float s = fmaxf(amax, 1e-4f) / 448.0f;  // IEEE division (no fast-math)
        if (pow2) {
            const uint32_t b = __float_as_uint(s);  // s is normal and positive
            if (b & 0x007FFFFFu) s = __uint_as_float((b & 0x7F800000u) + 0x00800000u);
        }
        const float y = __frcp_rn(s);
        float d[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) d[j] = quotient_rn(f[j], s, y);
        uint2 q;
        q.x = e4m3x2(d[0], d[1]) | (e4m3x2(d[2], d[3]) << 16);
        q.y = e4m3x2(d[4], d[5]) | (e4m3x2(d[6], d[7]) << 16);
        if (act) {
            reinterpret_cast<uint2*>(out_q)[b * 16 + l16] = q;
            if (l16 == 0) out_s[b] = s;
        }
    }
}

}  // namespace ep
