// combine.cu -- top-k weighted gather-reduce of expert outputs back into token order.
//
// "DeepSeek 开源周第二弹：DeepEP", section "DeepEP 的常规内核和低延迟内核": BF16 result
// merge; "deepseek-ai/DeepEP", section "典型工作流程": combine reduces the expert
// outputs back to where the tokens came from.  For token t, channel i:
//     acc = +0.0f;  for k = 0..K-1 with row_of[t, k] >= 0:
//         acc = fmaf(w[t, k], float(expert_out[row_of[t, k], i]), acc)
//     y[t, i] = bf16_rne(acc)
// The k order is fixed, so the result is bit-reproducible.
//
// Layout of the work: a CTA owns a slice of a token's row (blockIdx.y) and walks
// tokens t = blockIdx.x, blockIdx.x + gridDim.x, ...; each thread owns 8 channels
// (one 16-byte vector) and issues the loads of the token's valid rows for its
// channels (up to kBatch at a time) before it uses any, so up to 128 B per thread
// are in flight.  The K
// source rows are contiguous 14 KB rows (hidden 7168), so every warp reads whole
// 512-byte runs: the reads are coalesced and the traffic is the algorithmic
// minimum (K rows read once, one row written).  The rows and weights of the
// next token are prefetched while the current one is reduced.  In peer mode
// (partitions are the ranks of a node) the rows are read from the owner ranks'
// IPC-mapped expert outputs; the arithmetic and its order are the same.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kCombineMaxThreads = 512;
constexpr int64_t kPdlMaxEntries = 4096;  // (t, k) slots up to which the launch is programmatic
constexpr int kLoadBatch = 8;  // combine backward: slots handled per batch

// kBatch: row loads issued per thread before the first FMA.  The token's valid
// rows are compacted (k order kept) so a batch holds only rows that exist; sparse
// routings (one slot per partition, about half of them empty) use a batch of 4 and
// fewer registers, so three CTAs per SM and more loads in flight.
// kPeer: partitions are ranks; slot k's row is row_of[t, k] + peer_offset[e] in the
// expert outputs of the rank that owns e = topk_idx[t, k] (read over NVLink), or,
// for low-latency rows (row_of = e * cap + j), row ((e % Epp) * W + rank) * cap + j
// of rank e / Epp's padded outputs; the compaction records a pointer to each valid
// row instead of its index.
// kBySlot (deduplicated rows, slot k = rank k): slot k's row is row_of[t, k] +
// peer_offset[k] in rank k's outputs.  Lane k's offset and base address are the
// same for every token, so they are read once into shared memory, and the variant
// needs no expert ids: it fits three CTAs per SM without spilling.  Deduplicated
// normal workload: 57.3 us at two CTAs per SM, 53.0 us at three with a spilling
// generic peer variant, 51.5 us with the offsets in shared memory, 47.5 us with this
// variant -- the time of the one-GPU deduplicated combine.
template <int kBatch, bool kPeer, bool kBySlot = false>
__global__ void __launch_bounds__(kCombineMaxThreads, kBatch == 4 ? 3 : 2)
    combine_kernel(CombineParams p, int64_t vec_per_slice) {
    static_assert(kPeer || !kBySlot, "slot-indexed rows are a peer layout");
    pdl_wait();               // the previous kernel is complete (a no-op without the attribute)
    pdl_launch_dependents();  // the next kernel may be scheduled
    __shared__ int rows_sm[2][32];
    __shared__ const uint4* src_sm[kPeer ? 2 : 1][kPeer ? 32 : 1];
    __shared__ float w_sm[2][32];
    __shared__ int cnt_sm[2];
    const int tid = threadIdx.x;
    const int K = p.K;
    const int64_t T = p.T, V = p.H / 8;
    const int64_t v0 = static_cast<int64_t>(blockIdx.y) * vec_per_slice;
    const int64_t v1 = min(V, v0 + vec_per_slice);
    const uint4* eo = static_cast<const uint4*>(p.expert_out);
    uint4* y = static_cast<uint4*>(p.y);

    int nrow = -1;
    float nw = 1.0f;
    int64_t ne = -1;
    if (tid < K && static_cast<int64_t>(blockIdx.x) < T) {
        nrow = p.row_of[static_cast<int64_t>(blockIdx.x) * K + tid];
        if (p.topk_weights) nw = p.topk_weights[static_cast<int64_t>(blockIdx.x) * K + tid];
        if constexpr (kPeer)
            if (!kBySlot) ne = p.topk_idx[static_cast<int64_t>(blockIdx.x) * K + tid];
    }
    // deduplicated rows (slot k = rank k): lane k's row offset and base address are
    // the same for every token, so they are read once here instead of per token on
    // warp 0's set-up path
    __shared__ const uint4* slot_base_sm[kPeer ? 32 : 1];
    __shared__ int slot_off_sm[kPeer ? 32 : 1];
    if constexpr (kPeer)
        if (kBySlot && tid < K) {
            slot_off_sm[tid] = p.peer_offset[tid];
            slot_base_sm[tid] = static_cast<const uint4*>(p.peer_out[tid]);
        }
    __syncwarp();
    int buf = 0;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x, buf ^= 1) {
        if (tid < 32) {  // warp 0: lane k < K holds slot k
            int r = tid < K ? nrow : -1;
            const uint4* src = nullptr;
            if constexpr (kPeer) {
                // rows past the owner's buffer (or with an id the handle does not
                // match) are skipped
                if (kBySlot && r >= 0) {
                    const int64_t pr = static_cast<int64_t>(r) + slot_off_sm[tid];
                    if (pr < 0 || pr >= p.expert_out_rows) {
                        raise_status(p.status, kDevIndexRange);
                        r = -1;
                    } else {
                        src = slot_base_sm[tid] + pr * V;
                    }
                } else if (!kBySlot && r >= 0) {
                    const int at = ne >= 0 && ne < p.num_experts ? static_cast<int>(ne) : -1;
                    const int part = at >= 0 ? at / p.experts_per_partition : 0;
                    int64_t pr = -1;
                    if (at >= 0 && p.peer_ll_cap > 0) {
                        const int64_t c = p.peer_ll_cap;
                        const int64_t j = static_cast<int64_t>(r) - static_cast<int64_t>(at) * c;
                        const int64_t el = at - part * p.experts_per_partition;
                        if (j >= 0 && j < c) pr = (el * p.peer_world + p.peer_rank) * c + j;
                    } else if (at >= 0) {
                        pr = static_cast<int64_t>(r) + p.peer_offset[at];
                    }
                    if (pr < 0 || pr >= p.expert_out_rows) {
                        raise_status(p.status, kDevIndexRange);
                        r = -1;
                    } else {
                        src = static_cast<const uint4*>(p.peer_out[part]) + pr * V;
                    }
                }
            } else if (r >= 0 && static_cast<int64_t>(r) >= p.expert_out_rows) {
                raise_status(p.status, kDevIndexRange);
                r = -1;
            }
            const unsigned valid = __ballot_sync(0xffffffffu, r >= 0);
            if (r >= 0) {
                const int at = __popc(valid & ((1u << tid) - 1u));
                if constexpr (kPeer)
                    src_sm[buf][at] = src;
                else
                    rows_sm[buf][at] = r;
                w_sm[buf][at] = nw;
            }
            if (tid == 0) cnt_sm[buf] = __popc(valid);
            if (tid < K) {
                if (p.grad_w && blockIdx.y == 0)
                    p.grad_w[t * K + tid] = r >= 0 ? p.grad_recv_w[r] : 0.0f;
                const int64_t tn = t + gridDim.x;
                if (tn < T) {
                    nrow = p.row_of[tn * K + tid];
                    if (p.topk_weights) nw = p.topk_weights[tn * K + tid];
                    if constexpr (kPeer)
                        if (!kBySlot) ne = p.topk_idx[tn * K + tid];
                }
            }
        }
        __syncthreads();
        const int* rows = rows_sm[buf];
        const float* ws = w_sm[buf];
        const int m = cnt_sm[buf];
        for (int64_t v = v0 + tid; v < v1; v += blockDim.x) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
            for (int k0 = 0; k0 < m; k0 += kBatch) {
                uint4 d[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int k = k0 + u;
                    if constexpr (kPeer)
                        d[u] = k < m ? ld_stream_v4(src_sm[buf][k] + v) : make_uint4(0u, 0u, 0u, 0u);
                    else
                        d[u] = k < m ? ld_stream_v4(eo + static_cast<int64_t>(rows[k]) * V + v)
                                     : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int k = k0 + u;
                    if (k < m) {
                        const float w = ws[k];
                        acc[0] = __fmaf_rn(w, bf16_lo(d[u].x), acc[0]);
                        acc[1] = __fmaf_rn(w, bf16_hi(d[u].x), acc[1]);
                        acc[2] = __fmaf_rn(w, bf16_lo(d[u].y), acc[2]);
                        acc[3] = __fmaf_rn(w, bf16_hi(d[u].y), acc[3]);
                        acc[4] = __fmaf_rn(w, bf16_lo(d[u].z), acc[4]);
                        acc[5] = __fmaf_rn(w, bf16_hi(d[u].z), acc[5]);
                        acc[6] = __fmaf_rn(w, bf16_lo(d[u].w), acc[6]);
                        acc[7] = __fmaf_rn(w, bf16_hi(d[u].w), acc[7]);
                    }
                }
            }
            uint4 out;
            out.x = bf16x2_rn(acc[0], acc[1]);
            out.y = bf16x2_rn(acc[2], acc[3]);
            out.z = bf16x2_rn(acc[4], acc[5]);
            out.w = bf16x2_rn(acc[6], acc[7]);
            y[t * V + v] = out;
        }
        // rows_sm[buf] is rewritten two tokens later, after the next barrier
    }
}

// Backward of combine y[t] = sum_k w[t, k] * expert_out[row_of[t, k]]:
//   grad_expert_out[row, i] = bf16_rne(w[t, k] * grad_y[t, i])   (one fp32 multiply)
//   grad_topk_weights[t, k] = float(sum_i double(grad_y[t, i] * expert_out[row, i]))
// A product of two BF16 values is exact in fp32 (8 + 8 significant bits); the sum
// runs in fp64, which is exact -- and so independent of the summation order -- while
// the products span fewer than 37 binades.  One CTA per token row (grid-stride);
// each thread owns 8-channel vectors and issues the loads of up to 8 slots before
// using them; the per-slot dot products are reduced across the CTA in a fixed
// order (warp shuffles, then warps in index order).
constexpr int kBwdThreads = 448;

__global__ void __launch_bounds__(kBwdThreads) combine_backward_kernel(CombineBackwardParams p) {
    __shared__ int rows_sm[32];
    __shared__ float w_sm[32];
    __shared__ double red[kBwdThreads / 32][kLoadBatch];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int K = p.K;
    const int64_t T = p.T, V = p.H / 8;
    const uint4* gy = static_cast<const uint4*>(p.grad_y);
    const uint4* eo = static_cast<const uint4*>(p.expert_out);
    uint4* geo = static_cast<uint4*>(p.grad_expert_out);
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        if (tid < K) {
            int r = p.row_of[t * K + tid];
            if (r >= 0 && static_cast<int64_t>(r) >= p.expert_out_rows) {
                raise_status(p.status, kDevIndexRange);
                r = -1;
            }
            rows_sm[tid] = r;
            w_sm[tid] = p.topk_weights[t * K + tid];
        }
        __syncthreads();
        for (int k0 = 0; k0 < K; k0 += kLoadBatch) {
            double dot[kLoadBatch];
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u) dot[u] = 0.0;
            for (int64_t v = tid; v < V; v += blockDim.x) {
                const uint4 g = ld_stream_v4(gy + t * V + v);
                float gf[8];
                gf[0] = bf16_lo(g.x); gf[1] = bf16_hi(g.x); gf[2] = bf16_lo(g.y); gf[3] = bf16_hi(g.y);
                gf[4] = bf16_lo(g.z); gf[5] = bf16_hi(g.z); gf[6] = bf16_lo(g.w); gf[7] = bf16_hi(g.w);
                uint4 d[kLoadBatch];
#pragma unroll
                for (int u = 0; u < kLoadBatch; ++u) {
                    const int k = k0 + u;
                    const int r = k < K ? rows_sm[k] : -1;
                    d[u] = r >= 0 ? ld_stream_v4(eo + static_cast<int64_t>(r) * V + v)
                                  : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < kLoadBatch; ++u) {
                    const int k = k0 + u;
                    const int r = k < K ? rows_sm[k] : -1;
                    if (r < 0) continue;
                    float ef[8];
                    ef[0] = bf16_lo(d[u].x); ef[1] = bf16_hi(d[u].x);
                    ef[2] = bf16_lo(d[u].y); ef[3] = bf16_hi(d[u].y);
                    ef[4] = bf16_lo(d[u].z); ef[5] = bf16_hi(d[u].z);
                    ef[6] = bf16_lo(d[u].w); ef[7] = bf16_hi(d[u].w);
#pragma unroll
                    for (int j = 0; j < 8; ++j) dot[u] += static_cast<double>(__fmul_rn(gf[j], ef[j]));
                    const float w = w_sm[k];
                    uint4 o;
                    o.x = bf16x2_rn(__fmul_rn(w, gf[0]), __fmul_rn(w, gf[1]));
                    o.y = bf16x2_rn(__fmul_rn(w, gf[2]), __fmul_rn(w, gf[3]));
                    o.z = bf16x2_rn(__fmul_rn(w, gf[4]), __fmul_rn(w, gf[5]));
                    o.w = bf16x2_rn(__fmul_rn(w, gf[6]), __fmul_rn(w, gf[7]));
                    geo[static_cast<int64_t>(r) * V + v] = o;
                }
            }
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u) {
                double s = dot[u];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane == 0) red[warp][u] = s;
            }
            __syncthreads();
            if (tid < kLoadBatch && k0 + tid < K) {
                double s = 0.0;
                for (int w2 = 0; w2 < nwarps; ++w2) s += red[w2][tid];
                const int k = k0 + tid;
                p.grad_topk_weights[t * K + k] = rows_sm[k] >= 0 ? __double2float_rn(s) : 0.0f;
            }
            __syncthreads();
        }
    }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
    if (p.T == 0) return cudaSuccess;
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const int64_t V = p.H / 8;
    // slices of a row: at most kCombineMaxThreads vectors each, and enough
    // (token, slice) CTAs to cover every SM twice on small batches
    int64_t slices = (V + kCombineMaxThreads - 1) / kCombineMaxThreads;
    const int64_t want = (2LL * dev.num_sms + p.T - 1) / p.T;
    if (slices < want) slices = want;
    if (slices > V) slices = V;
    if (slices > 65535) slices = 65535;
    const int64_t per_slice = (V + slices - 1) / slices;
    slices = (V + per_slice - 1) / per_slice;
    int threads = static_cast<int>((per_slice + 31) / 32 * 32);
    if (threads > kCombineMaxThreads) threads = kCombineMaxThreads;
    const void* kernel =
        p.peer_out ? (p.peer_by_slot ? reinterpret_cast<const void*>(combine_kernel<4, true, true>)
                                     : reinterpret_cast<const void*>(combine_kernel<8, true>))
        : p.sparse ? reinterpret_cast<const void*>(combine_kernel<4, false>)
                   : reinterpret_cast<const void*>(combine_kernel<8, false>);
    const int per_sm = blocks_per_sm(kernel, dev.device, threads, 0);
    int64_t gx = (static_cast<int64_t>(per_sm) * dev.num_sms + slices - 1) / slices;
    if (gx > p.T) gx = p.T;
    if (gx < 1) gx = 1;
    if (gx > 2147483647LL) gx = 2147483647LL;
    // Decode-sized batches: a programmatic dependent launch, so the CTAs may be
    // scheduled while the previous kernel finishes (each waits for it with
    // griddepcontrol.wait before reading anything): the launch latency overlaps a
    // short predecessor (low-latency combine 3.6 -> 3.3 us per call).  Larger batches
    // launch once the previous kernel is complete: early CTAs slowed the dispatch
    // they overlapped (layout + dispatch + combine captured in one graph, normal
    // workload: 166.3 us per step with the early launch, 147.1 us without).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(slices));
    cfg.blockDim = dim3(threads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.T * static_cast<int64_t>(p.K) <= kPdlMaxEntries ? 1 : 0;
    if (p.peer_out && p.peer_by_slot)
        return cudaLaunchKernelEx(&cfg, combine_kernel<4, true, true>, p, per_slice);
    if (p.peer_out) return cudaLaunchKernelEx(&cfg, combine_kernel<8, true>, p, per_slice);
    if (p.sparse) return cudaLaunchKernelEx(&cfg, combine_kernel<4, false>, p, per_slice);
    return cudaLaunchKernelEx(&cfg, combine_kernel<8, false>, p, per_slice);
}

}  // namespace ep

namespace ep {

cudaError_t launch_combine_backward(const CombineBackwardParams& p, cudaStream_t stream) {
    if (p.T == 0) return cudaSuccess;
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const int64_t V = p.H / 8;
    int threads = static_cast<int>((V + 31) / 32 * 32);
    if (threads > kBwdThreads) threads = kBwdThreads;
    const int per_sm =
        blocks_per_sm(reinterpret_cast<const void*>(combine_backward_kernel), dev.device, threads, 0);
    int64_t grid = static_cast<int64_t>(per_sm) * dev.num_sms;
    if (grid > p.T) grid = p.T;
    combine_backward_kernel<<<static_cast<unsigned>(grid), threads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
