/*
 * ep_oracle.c -- plain, slow CPU statement of MoE token dispatch and combine.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file's library.  The CUDA library
 * never includes, links or calls it, and this file includes nothing of the
 * CUDA library: the two share no code.
 *
 * What is computed, and where it comes from:
 *
 *  - Dispatch sends every token's hidden vector to each expert it is routed
 *    to; combine gathers the expert outputs back to the token and merges them
 *    in BF16.  Pages: "DeepSeek 开源周第二弹：DeepEP —— 首个 MoE 模型训练和推理的
 *    EP 通信库" (m.youleyou.com), sections "DeepEP 的核心功能" (native FP8
 *    support) and "DeepEP 的常规内核和低延迟内核" (FP8 dispatch, BF16 result
 *    merge); deepseek.csdn.net/67bd3eb22e30c863900615cc, section "使用示例"
 *    (dispatch returns recv_x, recv_topk_idx, recv_topk_weights, handle).
 *  - The pages do not fix the FP8 format.  This library's reading: OCP FP8
 *    E4M3 (bias 7, largest finite 448, no infinities, NaN = S.1111.111), one
 *    fp32 scale per 1x128 block of channels, scale = max(amax, 1e-4) / 448 in
 *    fp32, q = e4m3(x / scale) with the fp32 quotient rounded to nearest-even
 *    and saturated to +-448.
 *  - The receive buffer is expert-major: expert ids ascending, then token
 *    index ascending, then top-k slot ascending (a stable counting sort of the
 *    (token, slot) pairs by expert id).  Logical partition p owns experts
 *    [p*E/P, (p+1)*E/P), so each partition's rows are one contiguous slice.
 *  - Combine: acc = +0.0f; for k = 0..K-1 with a valid row,
 *    acc = fmaf(w[t][k], float(expert_out[row][i]), acc); y = bf16_rne(acc).
 *  - Low-latency dispatch writes the same payload into a padded
 *    [E, capacity, H] tensor: slot j of (t, k) inside expert e is its stable
 *    rank among e's rows.  deepseek.csdn.net/67bd3eb22e30c863900615cc,
 *    section "推理解码阶段的应用": the buffer holds
 *    num_max_tokens * hidden * num_experts elements, so the capacity per
 *    expert is num_max_tokens.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fexcess-precision=standard
 * (no fast-math), so every float operation is a single IEEE-754 binary32
 * operation rounded to nearest-even, and fmaf is the fused multiply-add.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_INDEX_RANGE 1u /* a topk_idx / row outside its range was skipped */
#define ORACLE_CAPACITY 4u    /* a low-latency row did not fit its expert's capacity */

/* ---------------------------------------------------------------- BF16 -- */

/* BF16 is the upper half of a binary32 word: sign, 8 exponent bits, 7
 * mantissa bits.  Widening is exact. */
float oracle_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round binary32 to the nearest BF16, ties to the even mantissa.  For one
 * sign the magnitude order is the bit order, so the candidates are the
 * truncated pattern and the next pattern up; the dropped 16 bits decide. */
uint16_t oracle_bf16_from_f32(float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    if (isnan(v)) return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    uint32_t hi = u >> 16;
    uint32_t lo = u & 0xFFFFu;
    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u; /* may carry to inf */
    return (uint16_t)hi;
}

/* ---------------------------------------------------------------- E4M3 -- */

/* Decode an OCP E4M3 code: exponent field 0 is subnormal (m * 2^-9),
 * otherwise (1 + m/8) * 2^(E-7); S.1111.111 is NaN. */
float oracle_e4m3_to_f32(uint8_t c) {
    int sign = (c >> 7) & 1;
    int E = (c >> 3) & 0xF;
    int m = c & 7;
    double v;
    if (E == 15 && m == 7) return sign ? -NAN : NAN;
    if (E == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), E - 10);
    return (float)(sign ? -v : v);
}

/* Round a binary32 value to the nearest E4M3 value, ties to the even
 * mantissa, magnitudes above 448 saturated to 448 (no infinities in E4M3).
 * The sign of zero is kept.  All arithmetic is on exact binary64 values:
 * scaling by a power of two is exact and nearbyint() rounds to nearest-even
 * in the default rounding mode. */
uint8_t oracle_e4m3_from_f32(float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    uint8_t sign = (u >> 31) ? 0x80 : 0x00;
    if (isnan(v)) return (uint8_t)(sign | 0x7F);
    double a = fabs((double)v);
    if (a > 448.0) return (uint8_t)(sign | 0x7E); /* 0x7E = 1.75 * 2^8 = 448 */
    if (a < ldexp(1.0, -6)) {
        /* subnormal binade (and zero): spacing 2^-9; m = 8 lands on the
         * smallest normal 2^-6, whose code is also 8 (E = 1, mantissa 0). */
        double m = nearbyint(ldexp(a, 9));
        return (uint8_t)(sign | (uint8_t)m);
    }
    int e2;
    (void)frexp(a, &e2);      /* a = f * 2^e2, f in [0.5, 1) */
    int unb = e2 - 1;         /* a in [2^unb, 2^(unb+1)) */
    double m = nearbyint(ldexp(a, 3 - unb)); /* 8 + mantissa, in [8, 16] */
    int E = unb + 7;
    if (m == 16.0) { /* rounded up into the next binade */
        m = 8.0;
        E += 1;
    }
    return (uint8_t)(sign | (uint8_t)(E << 3) | (uint8_t)((int)m - 8));
}

/* Elementwise loops over the two encoders above (for exhaustive tests). */
void oracle_e4m3_from_f32_n(int64_t n, const float* v, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_from_f32(v[i]);
}

void oracle_bf16_from_f32_n(int64_t n, const float* v, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_from_f32(v[i]);
}

/* ------------------------------------------------------------ quantise -- */

/* Scale of one 1x128 block: max(amax, 1e-4) / 448, one binary32 division. */
float oracle_block_scale(float amax) {
    float a = fmaxf(amax, 1e-4f);
    return a / 448.0f;
}

/* Power-of-two scale of one block, for consumers that take scales as an 8-bit
 * exponent (UE8M0): the smallest power of two not below max(amax, 1e-4) / 448.
 * The quotient x / s is then an exact exponent shift and |x / s| <= 448.  The
 * pages fix no scale format; this is the library's optional second one. */
float oracle_block_scale_pow2(float amax) {
    float s = oracle_block_scale(amax);
    int e;
    double m = frexp((double)s, &e); /* s = m * 2^e, m in [0.5, 1) */
    if (m == 0.5) return s;          /* already a power of two */
    return (float)ldexp(1.0, e);
}

/* Quantise one BF16 row of H channels (H a multiple of 128) into E4M3 codes
 * and H/128 fp32 scales; pow2 selects the power-of-two scales. */
void oracle_quantize_row_mode(int64_t H, const uint16_t* x, uint8_t* q, float* scales, int pow2) {
    int64_t nb = H / 128;
    for (int64_t b = 0; b < nb; ++b) {
        float amax = 0.0f;
        for (int i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(oracle_bf16_to_f32(x[b * 128 + i])));
        float s = pow2 ? oracle_block_scale_pow2(amax) : oracle_block_scale(amax);
        for (int i = 0; i < 128; ++i) {
            float xv = oracle_bf16_to_f32(x[b * 128 + i]);
            q[b * 128 + i] = oracle_e4m3_from_f32(xv / s);
        }
        scales[b] = s;
    }
}

void oracle_quantize_row(int64_t H, const uint16_t* x, uint8_t* q, float* scales) {
    oracle_quantize_row_mode(H, x, q, scales, 0);
}

/* -------------------------------------------------------------- layout -- */

/* Routing layout of topk_idx[T][K] (-1 = masked slot).
 *   num_tokens_per_expert[e]     rows routed to expert e
 *   is_token_in_partition[t][p]  1 if token t names any expert of partition p
 *   num_tokens_per_partition[p]  number of distinct tokens with is_token_in_partition = 1
 *   expert_offset[E+1]           exclusive prefix sum of num_tokens_per_expert
 *   row_of[t][k]                 receive row of (t, k), -1 if masked
 *   src_of[row]                  t*K + k for each of the num_recv rows
 * An index outside [-1, E) is skipped like a masked slot and reported. */
uint32_t oracle_layout(int64_t T, int32_t K, int32_t E, int32_t P, const int64_t* topk_idx,
                       int32_t* num_tokens_per_expert, int32_t* num_tokens_per_partition,
                       uint8_t* is_token_in_partition, int32_t* expert_offset, int32_t* row_of,
                       int32_t* src_of, int32_t* num_recv) {
    uint32_t status = 0;
    int32_t epp = E / P;
    int32_t* seen = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int32_t e = 0; e < E; ++e) num_tokens_per_expert[e] = 0;
    for (int32_t p = 0; p < P; ++p) num_tokens_per_partition[p] = 0;
    for (int64_t i = 0; i < T * P; ++i) is_token_in_partition[i] = 0;

    for (int64_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[t * K + k];
            if (e == -1) continue;
            if (e < 0 || e >= E) {
                status |= ORACLE_INDEX_RANGE;
                continue;
            }
            num_tokens_per_expert[e] += 1;
            is_token_in_partition[t * P + e / epp] = 1;
        }
    }
    for (int64_t t = 0; t < T; ++t)
        for (int32_t p = 0; p < P; ++p) num_tokens_per_partition[p] += is_token_in_partition[t * P + p];

    expert_offset[0] = 0;
    for (int32_t e = 0; e < E; ++e) expert_offset[e + 1] = expert_offset[e] + num_tokens_per_expert[e];
    *num_recv = expert_offset[E];

    for (int64_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[t * K + k];
            if (e < 0 || e >= E) {
                row_of[t * K + k] = -1;
                continue;
            }
            int32_t row = expert_offset[e] + seen[e];
            seen[e] += 1;
            row_of[t * K + k] = row;
            src_of[row] = (int32_t)(t * K + k);
        }
    }
    free(seen);
    return status;
}

/* ------------------------------------------------------------ dispatch -- */

/* Copy every token to the rows the layout gave it.
 *   quant = 1: recv_x is E4M3 [rows][H], recv_scales fp32 [rows][H/128]
 *   quant = 2: the same with power-of-two scales (oracle_block_scale_pow2)
 *   quant = 0: recv_x is the BF16 row, bit for bit [rows][H]; recv_scales unused
 *   recv_topk_idx[row]     = local expert id e - p*E/P of the row's expert
 *   recv_topk_weights[row] = topk_weights[t][k]                              */
uint32_t oracle_dispatch(int64_t T, int64_t H, int32_t K, int32_t E, int32_t P, int32_t quant,
                         const uint16_t* x, const int64_t* topk_idx, const float* topk_weights,
                         const int32_t* row_of, uint8_t* recv_x, float* recv_scales,
                         int32_t* recv_topk_idx, float* recv_topk_weights) {
    int32_t epp = E / P;
    int64_t nb = H / 128;
    uint8_t* q = (uint8_t*)malloc((size_t)H);
    float* s = (float*)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    for (int64_t t = 0; t < T; ++t) {
        if (quant >= 1) oracle_quantize_row_mode(H, x + t * H, q, s, quant == 2);
        for (int32_t k = 0; k < K; ++k) {
            int32_t row = row_of[t * K + k];
            if (row < 0) continue;
            int64_t e = topk_idx[t * K + k];
            if (quant >= 1) {
                memcpy(recv_x + (int64_t)row * H, q, (size_t)H);
                memcpy(recv_scales + (int64_t)row * nb, s, sizeof(float) * (size_t)nb);
            } else {
                memcpy(recv_x + (int64_t)row * H * 2, x + t * H, (size_t)H * 2);
            }
            recv_topk_idx[row] = (int32_t)(e - (e / epp) * epp);
            recv_topk_weights[row] = topk_weights[t * K + k];
        }
    }
    free(q);
    free(s);
    return 0;
}

/* Stand-in for the expert computation in tests and benchmarks: the expert
 * returns its input.  FP8 rows are dequantised with one binary32 multiply
 * q * scale and rounded to BF16; BF16 rows are passed through. */
void oracle_identity_expert(int64_t R, int64_t H, int32_t quant, const uint8_t* recv_x,
                            const float* recv_scales, uint16_t* expert_out) {
    int64_t nb = H / 128;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t i = 0; i < H; ++i) {
            if (quant >= 1) {
                float v = oracle_e4m3_to_f32(recv_x[r * H + i]) * recv_scales[r * nb + i / 128];
                expert_out[r * H + i] = oracle_bf16_from_f32(v);
            } else {
                uint16_t b;
                memcpy(&b, recv_x + (r * H + i) * 2, 2);
                expert_out[r * H + i] = b;
            }
        }
    }
}

/* ------------------------------------------------------------- combine -- */

/* y[t][i] = bf16_rne( fmaf chain over k = 0..K-1 of w[t][k] * expert_out[row_of[t][k]][i] ),
 * starting from +0.0f and skipping masked slots (row -1).  A row outside
 * [0, expert_rows) is skipped and reported. */
uint32_t oracle_combine(int64_t T, int64_t H, int32_t K, const uint16_t* expert_out,
                        int64_t expert_rows, const int32_t* row_of, const float* topk_weights,
                        uint16_t* y) {
    uint32_t status = 0;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < H; ++i) {
            float acc = 0.0f;
            for (int32_t k = 0; k < K; ++k) {
                int32_t row = row_of[t * K + k];
                if (row < 0) continue;
                if ((int64_t)row >= expert_rows) {
                    status |= ORACLE_INDEX_RANGE;
                    continue;
                }
                float v = oracle_bf16_to_f32(expert_out[(int64_t)row * H + i]);
                acc = fmaf(topk_weights[t * K + k], v, acc);
            }
            y[t * H + i] = oracle_bf16_from_f32(acc);
        }
    }
    return status;
}

/* ------------------------------------------------------ low latency ----- */

/* Low-latency dispatch into a padded [E][cap][H] E4M3 tensor with
 * [E][cap][H/128] scales.  The slot of (t, k) inside expert e is the number
 * of earlier (t', k') routed to e (token-major, then k), the same order as the
 * normal layout.  A row that would land at slot >= cap is dropped and
 * reported.  recv_expert_count[e] = rows written to expert e.
 * ll_row_of[t][k] = e*cap + slot (-1 if masked or dropped);
 * ll_src_of[e*cap + slot] = t*K + k.  Unused slots are not written. */
uint32_t oracle_ll_dispatch(int64_t T, int64_t H, int32_t K, int32_t E, int32_t cap,
                            const uint16_t* x, const int64_t* topk_idx, uint8_t* recv_x,
                            float* recv_scales, int32_t* recv_expert_count, int32_t* ll_row_of,
                            int32_t* ll_src_of) {
    uint32_t status = 0;
    int64_t nb = H / 128;
    int32_t* seen = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    uint8_t* q = (uint8_t*)malloc((size_t)H);
    float* s = (float*)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    for (int64_t t = 0; t < T; ++t) {
        oracle_quantize_row(H, x + t * H, q, s);
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[t * K + k];
            ll_row_of[t * K + k] = -1;
            if (e == -1) continue;
            if (e < 0 || e >= E) {
                status |= ORACLE_INDEX_RANGE;
                continue;
            }
            int32_t j = seen[e];
            seen[e] += 1;
            if (j >= cap) {
                status |= ORACLE_CAPACITY;
                continue;
            }
            int64_t row = e * (int64_t)cap + j;
            memcpy(recv_x + row * H, q, (size_t)H);
            memcpy(recv_scales + row * nb, s, sizeof(float) * (size_t)nb);
            ll_row_of[t * K + k] = (int32_t)row;
            ll_src_of[row] = (int32_t)(t * K + k);
        }
    }
    for (int32_t e = 0; e < E; ++e) recv_expert_count[e] = seen[e] < cap ? seen[e] : cap;
    free(seen);
    free(q);
    free(s);
    return status;
}

/* ------------------------------------------------------------ backward -- */

/* Backward of dispatch ("deepseek-ai/DeepEP" (agentlenshq.com), section
 * "典型工作流程": combine "or the backward helpers" reduce results back).  Every
 * receive row is a copy of its token, so the gradient of x sums the gradients of
 * the token's rows:
 *   grad_x[t][i] = bf16_rne( +0.0f + grad_recv_x[row_of[t][0]][i] + ... ), rows in
 *   k order, masked slots skipped;
 * and recv_topk_weights[row] = topk_weights[t][k] gives
 *   grad_topk_weights[t][k] = grad_recv_topk_weights[row_of[t][k]] (0 if masked).
 * grad_recv_topk_weights / grad_topk_weights may be NULL. */
uint32_t oracle_dispatch_backward(int64_t T, int64_t H, int32_t K, const uint16_t* grad_recv_x,
                                  int64_t rows, const int32_t* row_of,
                                  const float* grad_recv_topk_weights, uint16_t* grad_x,
                                  float* grad_topk_weights) {
    uint32_t status = 0;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < H; ++i) {
            float acc = 0.0f;
            for (int32_t k = 0; k < K; ++k) {
                int32_t row = row_of[t * K + k];
                if (row < 0) continue;
                if ((int64_t)row >= rows) {
                    status |= ORACLE_INDEX_RANGE;
                    continue;
                }
                acc = acc + oracle_bf16_to_f32(grad_recv_x[(int64_t)row * H + i]);
            }
            grad_x[t * H + i] = oracle_bf16_from_f32(acc);
        }
        if (grad_recv_topk_weights && grad_topk_weights) {
            for (int32_t k = 0; k < K; ++k) {
                int32_t row = row_of[t * K + k];
                grad_topk_weights[t * K + k] =
                    (row >= 0 && (int64_t)row < rows) ? grad_recv_topk_weights[row] : 0.0f;
            }
        }
    }
    return status;
}

/* Backward of combine y[t] = sum_k w[t][k] * expert_out[row_of[t][k]]:
 *   grad_expert_out[row_of[t][k]][i] = bf16_rne( w[t][k] * float(grad_y[t][i]) )
 *     (one binary32 multiply; rows no slot points at are not written);
 *   grad_topk_weights[t][k] = float( sum over i = 0..H-1 of
 *     (double)grad_y[t][i] * (double)expert_out[row][i] ), 0 for masked slots.
 * Each product of two BF16 values is exact in binary32 (8 + 8 significant bits)
 * and the sum runs in binary64, so while the products' magnitudes span fewer
 * than 37 binades the sum is exact and its rounding to binary32 does not depend
 * on the order of the terms. */
uint32_t oracle_combine_backward(int64_t T, int64_t H, int32_t K, const uint16_t* grad_y,
                                 const uint16_t* expert_out, int64_t rows, const int32_t* row_of,
                                 const float* topk_weights, uint16_t* grad_expert_out,
                                 float* grad_topk_weights) {
    uint32_t status = 0;
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
            int32_t row = row_of[t * K + k];
            double dot = 0.0;
            int valid = row >= 0 && (int64_t)row < rows;
            if (row >= 0 && !valid) status |= ORACLE_INDEX_RANGE;
            if (valid) {
                float w = topk_weights[t * K + k];
                for (int64_t i = 0; i < H; ++i) {
                    float g = oracle_bf16_to_f32(grad_y[t * H + i]);
                    float e = oracle_bf16_to_f32(expert_out[(int64_t)row * H + i]);
                    grad_expert_out[(int64_t)row * H + i] = oracle_bf16_from_f32(w * g);
                    dot += (double)g * (double)e;
                }
            }
            grad_topk_weights[t * K + k] = valid ? (float)dot : 0.0f;
        }
    }
    return status;
}

/* ------------------------------------------------- deduplicated dispatch -- */

/* Dispatch with one receive row per (token, partition) instead of one per
 * (token, expert): DeepEP's normal kernels send a token once to each rank that
 * holds any of its experts, with the list of that rank's experts and weights
 * (deepseek.csdn.net/67bd3eb22e30c863900615cc, section "使用示例": dispatch
 * returns recv_x, recv_topk_idx, recv_topk_weights; "DeepSeek 开源周第二弹：DeepEP",
 * section "DeepEP 的常规内核和低延迟内核": top-4 groups of top-8 experts).
 * Partitions stand for the ranks: partition p owns experts [p*E/P, (p+1)*E/P).
 *   prow_of[t][p]  row of (t, p): partition-major, token ascending; -1 if token t
 *                  names no expert of partition p
 *   part_count[p], part_offset[P+1], src_tok[row] = t, *num_rows
 *   recv_x[row]    the token's row (E4M3 + 1x128 scales, or BF16 bits)
 *   recv_topk_idx[row][k]     e - p*E/P if topk_idx[t][k] = e lies in p, else -1
 *   recv_topk_weights[row][k] topk_weights[t][k] for those k, else 0
 * Ids outside [-1, E) are skipped and reported. */
uint32_t oracle_dispatch_dedup(int64_t T, int64_t H, int32_t K, int32_t E, int32_t P,
                               int32_t quant, const uint16_t* x, const int64_t* topk_idx,
                               const float* topk_weights, int32_t* prow_of, int32_t* part_count,
                               int32_t* part_offset, int32_t* src_tok, int32_t* num_rows,
                               uint8_t* recv_x, float* recv_scales, int32_t* recv_topk_idx,
                               float* recv_topk_weights) {
    uint32_t status = 0;
    int32_t epp = E / P;
    int64_t nb = H / 128;
    uint8_t* in_part = (uint8_t*)calloc((size_t)(T * P > 0 ? T * P : 1), 1);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[t * K + k];
            if (e == -1) continue;
            if (e < 0 || e >= E) {
                status |= ORACLE_INDEX_RANGE;
                continue;
            }
            in_part[t * P + e / epp] = 1;
        }
    }
    for (int32_t p = 0; p < P; ++p) {
        part_count[p] = 0;
        for (int64_t t = 0; t < T; ++t) part_count[p] += in_part[t * P + p];
    }
    part_offset[0] = 0;
    for (int32_t p = 0; p < P; ++p) part_offset[p + 1] = part_offset[p] + part_count[p];
    *num_rows = part_offset[P];
    uint8_t* q = (uint8_t*)malloc((size_t)H);
    float* s = (float*)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    for (int32_t p = 0; p < P; ++p) {
        int32_t row = part_offset[p];
        for (int64_t t = 0; t < T; ++t) {
            if (!in_part[t * P + p]) {
                prow_of[t * P + p] = -1;
                continue;
            }
            prow_of[t * P + p] = row;
            src_tok[row] = (int32_t)t;
            if (quant >= 1) {
                oracle_quantize_row_mode(H, x + t * H, q, s, quant == 2);
                memcpy(recv_x + (int64_t)row * H, q, (size_t)H);
                memcpy(recv_scales + (int64_t)row * nb, s, sizeof(float) * (size_t)nb);
            } else {
                memcpy(recv_x + (int64_t)row * H * 2, x + t * H, (size_t)H * 2);
            }
            for (int32_t k = 0; k < K; ++k) {
                int64_t e = topk_idx[t * K + k];
                int in = e >= 0 && e < E && e / epp == p;
                recv_topk_idx[(int64_t)row * K + k] = in ? (int32_t)(e - (int64_t)p * epp) : -1;
                recv_topk_weights[(int64_t)row * K + k] = in ? topk_weights[t * K + k] : 0.0f;
            }
            row += 1;
        }
    }
    free(in_part);
    free(q);
    free(s);
    return status;
}

/* Stand-in for a partition's experts in tests and benchmarks of the
 * deduplicated path: every expert returns its input, and the partition reduces
 * its experts' outputs with their weights before sending the row back, so
 *   out[row][i] = bf16_rne( fmaf chain over k with recv_topk_idx[row][k] >= 0 of
 *                 recv_topk_weights[row][k] * v[i] ),  v = the dequantised row
 *   (q * scale in one binary32 multiply, or the BF16 row). */
void oracle_partition_identity(int64_t rows, int64_t H, int32_t K, int32_t quant,
                               const uint8_t* recv_x, const float* recv_scales,
                               const int32_t* recv_topk_idx, const float* recv_topk_weights,
                               uint16_t* out) {
    int64_t nb = H / 128;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t i = 0; i < H; ++i) {
            float v;
            if (quant >= 1) {
                v = oracle_e4m3_to_f32(recv_x[r * H + i]) * recv_scales[r * nb + i / 128];
            } else {
                uint16_t b;
                memcpy(&b, recv_x + (r * H + i) * 2, 2);
                v = oracle_bf16_to_f32(b);
            }
            float acc = 0.0f;
            for (int32_t k = 0; k < K; ++k) {
                if (recv_topk_idx[r * K + k] < 0) continue;
                acc = fmaf(recv_topk_weights[r * K + k], v, acc);
            }
            out[r * H + i] = oracle_bf16_from_f32(acc);
        }
    }
}

/* Combine of the deduplicated path: each partition returns one already-weighted
 * row per token, so y[t][i] = bf16_rne( +0.0f + out[prow_of[t][0]][i] + ... ) over
 * the partitions the token touched, in partition order (binary32 adds). */
uint32_t oracle_combine_dedup(int64_t T, int64_t H, int32_t P, const uint16_t* part_out,
                              int64_t rows, const int32_t* prow_of, uint16_t* y) {
    uint32_t status = 0;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < H; ++i) {
            float acc = 0.0f;
            for (int32_t p = 0; p < P; ++p) {
                int32_t row = prow_of[t * P + p];
                if (row < 0) continue;
                if ((int64_t)row >= rows) {
                    status |= ORACLE_INDEX_RANGE;
                    continue;
                }
                acc = acc + oracle_bf16_to_f32(part_out[(int64_t)row * H + i]);
            }
            y[t * H + i] = oracle_bf16_from_f32(acc);
        }
    }
    return status;
}

/* ---------------------------------------------------- redundant experts -- */
/*
 * Expert replication for load balancing.  Pages: "deepseek-ai/DeepEP"
 * (agentlenshq.com), section "主要特性" (redundant-expert support through
 * lb_prefetch_weights / lb_reduce_grads) and section "典型工作流程", step 5
 * (optionally replicate heavily loaded experts across NVLink-connected GPUs);
 * the page's opening paragraph adds that the kernels prefetch expert weights
 * and reduce redundant gradients.  The pages name the calls and their purpose
 * only.  This library's reading, with one GPU's expert slots standing for the
 * ranks' slots:
 *  - primary_of[s] is the slot holding the authoritative copy of slot s's
 *    expert; a primary names itself, a replica names its primary.
 *  - prefetch_weights: every replica slot receives a byte copy of its
 *    primary's weight blob; primaries are left as they are.
 *  - reduce_grads: the fp32 gradients of a primary and its replicas are summed
 *    in ascending slot order (the first slot's value, then one binary32 add per
 *    further slot), and the sum is written to every slot of the group, so all
 *    copies apply the same update.  A slot whose primary_of entry is out of
 *    range, or names a slot that is not a primary, is skipped (status bit 1).
 */
static int oracle_lb_valid(int32_t S, const int32_t* primary_of, int32_t s) {
    int32_t q = primary_of[s];
    return q >= 0 && q < S && primary_of[q] == q;
}

uint32_t oracle_lb_prefetch_weights(int32_t S, int64_t nbytes, const int32_t* primary_of,
                                    uint8_t* weights) {
    uint32_t status = 0;
    for (int32_t s = 0; s < S; ++s) {
        if (!oracle_lb_valid(S, primary_of, s)) {
            status |= ORACLE_INDEX_RANGE;
            continue;
        }
        int32_t q = primary_of[s];
        if (q != s) memcpy(weights + (int64_t)s * nbytes, weights + (int64_t)q * nbytes, (size_t)nbytes);
    }
    return status;
}

uint32_t oracle_lb_reduce_grads(int32_t S, int64_t n, const int32_t* primary_of, float* grads) {
    uint32_t status = 0;
    float* acc = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    for (int32_t s = 0; s < S; ++s)
        if (!oracle_lb_valid(S, primary_of, s)) status |= ORACLE_INDEX_RANGE;
    for (int32_t q = 0; q < S; ++q) {
        if (primary_of[q] != q) continue; /* q is not a primary */
        int first = 1;
        for (int32_t s = 0; s < S; ++s) { /* ascending slot order */
            if (!oracle_lb_valid(S, primary_of, s) || primary_of[s] != q) continue;
            const float* g = grads + (int64_t)s * n;
            for (int64_t i = 0; i < n; ++i) acc[i] = first ? g[i] : acc[i] + g[i];
            first = 0;
        }
        for (int32_t s = 0; s < S; ++s) {
            if (!oracle_lb_valid(S, primary_of, s) || primary_of[s] != q) continue;
            memcpy(grads + (int64_t)s * n, acc, sizeof(float) * (size_t)n);
        }
    }
    free(acc);
    return status;
}
