// low_latency.cu -- low-latency dispatch for small decode batches, one fused kernel.
//
// deepseek.csdn.net/67bd3eb22e30c863900615cc, section "推理解码阶段的应用":
// low_latency_dispatch(hidden_states, topk_idx, num_max_tokens, num_experts) returns
// recv_hidden_states and recv_expert_count; the buffer holds
// num_max_tokens * hidden * num_experts elements, i.e. num_max_tokens rows per
// expert.  "DeepSeek 开源周第二弹：DeepEP", section "DeepEP 的常规内核和低延迟内核":
// 128-token decode batches, FP8 dispatch.
//
// One kernel does everything the normal path does in its layout and dispatch
// kernels; each token's row is split into slices, one CTA per (token, slice):
//   - the slice's bulk load is issued first, so its latency overlaps the rest;
//   - slot of (t, k) in expert e = number of earlier (t', k') routed to e: a
//     shared-memory histogram of the earlier tokens' ids (the batch is small, the
//     prefix is L2-hot) plus equal ids in the token's own earlier slots;
//     the order is the normal layout's, so slot j of e holds normal row
//     expert_offset[e] + j;
//   - CTA 0 also histograms all T*K ids into recv_expert_count;
//   - quantise the slice (same arithmetic as the normal FP8 path) and bulk-store it
//     into slot e * num_max_tokens + j of each destination expert.
// Peer mode (template parameter kPeer; partitions are the ranks of a node, as in
// DeepEP's low-latency kernels, whose receive buffer is [local experts, ranks *
// num_max_tokens, hidden]): source rank s stores slot j of expert e into row
// ((e % Epp) * W + s) * num_max_tokens + j of rank e / Epp's buffer and its count of
// e into entry (e % Epp) * W + s of that rank's count table, so no counts have to be
// exchanged first.  The handle stays local (e * num_max_tokens + j).
#include "ep_device.cuh"
#include "ep_internal.h"
#include "ep_quant.cuh"

namespace ep {

namespace {

constexpr int kLLMaxThreads = 256;
constexpr int kPrefixBatch = 8;  // topk_idx loads in flight per thread

// Shared memory of one (token, slice) CTA: the slice's BF16 input, its E4M3 codes
// and scales, an mbarrier, the token's K rows / slot counters / ids, and (CTA 0
// only) the expert histogram.
struct LLSmem {
    uint32_t in_bytes, q_bytes, s_bytes;
    uint32_t off_q, off_s, off_bar, off_rows, off_cnt, off_eid, off_hist, total;
};

__host__ __device__ inline LLSmem ll_smem(int nbs, int32_t E) {
    LLSmem s;
    s.in_bytes = static_cast<uint32_t>(nbs) * 256u;
    s.q_bytes = static_cast<uint32_t>(nbs) * 128u;
    s.s_bytes = (static_cast<uint32_t>(nbs) * 4u + 15u) & ~15u;
    s.off_q = s.in_bytes;
    s.off_s = s.off_q + s.q_bytes;
    s.off_bar = s.off_s + s.s_bytes;
    s.off_rows = s.off_bar + 16u;
    s.off_cnt = s.off_rows + 4u * 32u;
    s.off_eid = s.off_cnt + 4u * 32u;
    s.off_hist = s.off_eid + 8u * 32u;
    s.total = s.off_hist + 4u * static_cast<uint32_t>(E);
    return s;
}

// Where slot row (= e * cap + j) of expert e goes: the local padded buffer, or in peer
// mode rank e / epp's buffer at ((e % epp) * world + rank) * cap + j.
template <bool kPeer>
__device__ __forceinline__ int64_t ll_dest(const LowLatencyDispatchParams& p, int row, int64_t e,
                                           uint8_t*& x, float*& s) {
    if constexpr (kPeer) {
        const int q = static_cast<int>(e) / p.epp;
        const int64_t j = row - e * p.cap;
        x = static_cast<uint8_t*>(p.peer_recv_x[q]);
        s = p.peer_recv_scales[q];
        return (static_cast<int64_t>(static_cast<int>(e) - q * p.epp) * p.world + p.rank) * p.cap + j;
    } else {
        x = static_cast<uint8_t*>(p.recv_x);
        s = p.recv_scales;
        return row;
    }
}

// grid = (T, S): CTA (t, y) handles token t's 128-channel blocks
// [y * nbs, min(nb, (y + 1) * nbs)).  Every slice computes the token's slots (the
// prefix is short and L2-hot); slice 0 also writes the handle; CTA (0, 0) writes
// recv_expert_count.
template <bool kPeer>
__global__ void __launch_bounds__(kLLMaxThreads) ll_dispatch_kernel(LowLatencyDispatchParams p,
                                                                    int nbs) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int64_t H = p.H;
    const int K = p.K, E = p.E, cap = p.cap, nb = static_cast<int>(H >> 7);
    const LLSmem L = ll_smem(nbs, E);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L.off_bar);
    int* rows_sm = reinterpret_cast<int*>(sm + L.off_rows);
    int* cnt_sm = reinterpret_cast<int*>(sm + L.off_cnt);
    int64_t* eid_sm = reinterpret_cast<int64_t*>(sm + L.off_eid);
    int* hist = reinterpret_cast<int*>(sm + L.off_hist);
    uint8_t* out_q = sm + L.off_q;
    float* out_s = reinterpret_cast<float*>(sm + L.off_s);
    const int64_t t = blockIdx.x;
    const int y = blockIdx.y;
    const int b0 = y * nbs;
    const int nbl = min(nb, b0 + nbs) - b0;  // blocks in this slice (>= 1)
    const bool head = (y == 0);
    const bool all = (t == 0 && y == 0);
    // scales go out by bulk copy when every row's slice of them is 16-byte aligned
    const bool scale_bulk = (nb % 4 == 0) && (nbs % 4 == 0) && (nbl % 4 == 0);

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nbl) * 256u);
        bulk_load(sm, static_cast<const uint8_t*>(p.x) + t * H * 2 + static_cast<int64_t>(b0) * 256,
                  static_cast<uint32_t>(nbl) * 256u, bar);
    }
    // slot of (t, k) = pairs (t', k') < (t, k) in (token, k) order with the same
    // expert: a histogram of the ids of the earlier tokens (shared-memory atomics,
    // kPrefixBatch loads in flight per thread; the first batch is issued before the
    // histogram is cleared, so its latency overlaps the barrier), plus the equal ids
    // among the token's own earlier slots.  CTA (0, 0) -- token 0, no earlier tokens
    // -- histograms the whole batch instead, for recv_expert_count.
    const int64_t base = t * K;
    const int64_t upto = all ? p.T * K : base;
    const int64_t stride = static_cast<int64_t>(blockDim.x);
    int64_t v[kPrefixBatch];
#pragma unroll
    for (int u = 0; u < kPrefixBatch; ++u) {
        const int64_t j = tid + u * stride;
        v[u] = j < upto ? p.topk_idx[j] : -1;
    }
    if (tid < K) eid_sm[tid] = p.topk_idx[t * K + tid];
    for (int e = tid; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    for (int64_t j0 = tid;; j0 += kPrefixBatch * stride) {
#pragma unroll
        for (int u = 0; u < kPrefixBatch; ++u)
            if (v[u] >= 0 && v[u] < E) atomicAdd(&hist[v[u]], 1);
        const int64_t jn = j0 + kPrefixBatch * stride;
        if (jn >= upto) break;
#pragma unroll
        for (int u = 0; u < kPrefixBatch; ++u) {
            const int64_t j = jn + u * stride;
            v[u] = j < upto ? p.topk_idx[j] : -1;
        }
    }
    __syncthreads();
    if (tid < K) {
        const int64_t e = eid_sm[tid];
        int same = 0;  // equal ids in this token's earlier slots
        for (int k = 0; k < tid; ++k) same += eid_sm[k] == e ? 1 : 0;
        cnt_sm[tid] = (t == 0 || e < 0 || e >= E ? 0 : hist[e]) + same;
    }
    __syncthreads();
    if (tid < K) {
        const int64_t e = eid_sm[tid];
        int row = -1;
        if (e != -1 && (e < 0 || e >= E)) {
            if (head) raise_status(p.status, kDevIndexRange);
        } else if (e >= 0) {
            const int j = cnt_sm[tid];
            if (j < cap)
                row = static_cast<int>(e * cap + j);
            else if (head)
                raise_status(p.status, kDevCapacity);
        }
        rows_sm[tid] = row;
        if (head) {
            p.row_of[base + tid] = row;
            if (row >= 0) p.src_of[row] = static_cast<int32_t>(base + tid);
        }
    }
    if (all) {
        for (int e = tid; e < E; e += blockDim.x) {
            if constexpr (kPeer)
                p.peer_recv_count[e / p.epp][(e % p.epp) * p.world + p.rank] = min(hist[e], cap);
            else
                p.recv_expert_count[e] = min(hist[e], cap);
        }
    }

    const bool ok = mbar_wait_bounded(bar, 0, p.timeout_ns);
    if (!__syncthreads_and(ok)) {
        if (tid == 0) {
            raise_status(p.status, kDevTimeout);
            mbar_wait_bounded(bar, 0, kDefaultTimeoutNs);  // let the load land before exiting
        }
        return;
    }
    quantize_row_fp8(sm, out_q, out_s, nbl, warp, nwarps, lane);
    fence_proxy_async_smem();
    __syncthreads();
    if (warp == 0 && lane < K) {
        const int row = rows_sm[lane];
        if (row >= 0) {
            uint8_t* dx;
            float* ds;
            const int64_t r = ll_dest<kPeer>(p, row, eid_sm[lane], dx, ds);
            bulk_store(dx + r * H + static_cast<int64_t>(b0) * 128, out_q,
                       static_cast<uint32_t>(nbl) * 128u);
            if (scale_bulk)
                bulk_store(ds + r * nb + b0, out_s, static_cast<uint32_t>(nbl) * 4u);
        }
        bulk_commit();
    }
    if (!scale_bulk) {
        for (int idx = tid; idx < K * nbl; idx += blockDim.x) {
            const int k = idx / nbl, b = idx - k * nbl;
            const int row = rows_sm[k];
            if (row >= 0) {
                uint8_t* dx;
                float* ds;
                const int64_t r = ll_dest<kPeer>(p, row, eid_sm[k], dx, ds);
                ds[r * nb + b0 + b] = out_s[b];
            }
        }
    }
    if (warp == 0 && lane < K) bulk_wait_read<0>();  // staged slice read: the CTA may exit
}

// Peer mode with no tokens: this rank's count of every expert is zero.
__global__ void ll_peer_zero_counts_kernel(LowLatencyDispatchParams p) {
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        p.peer_recv_count[e / p.epp][(e % p.epp) * p.world + p.rank] = 0;
}

__global__ void wait_probe_kernel(uint32_t* status, const volatile uint32_t* flag,
                                  uint64_t timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    // (1) a flag nothing sets
    const uint64_t t0 = globaltimer_ns();
    bool seen = false;
    while (!(seen = (*flag != 0u))) {
        if (globaltimer_ns() - t0 > timeout_ns) break;
    }
    if (!seen) raise_status(status, kDevTimeout);
    // (2) an mbarrier waiting for 16 transaction bytes no copy will deliver
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, 16u);
    if (!mbar_wait_bounded(&bar, 0, timeout_ns)) raise_status(status, kDevTimeout);
}

}  // namespace

cudaError_t launch_ll_dispatch(const LowLatencyDispatchParams& p, cudaStream_t stream) {
    if (p.T == 0) {
        // no tokens: every expert received nothing
        if (p.peer_recv_x) {
            ll_peer_zero_counts_kernel<<<1, 256, 0, stream>>>(p);
            return cudaGetLastError();
        }
        return cudaMemsetAsync(p.recv_expert_count, 0, sizeof(int32_t) * p.E, stream);
    }
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    // slices per token: enough (token, slice) CTAs to cover every SM about four
    // times, a multiple of 4 blocks per slice where possible (bulk scale stores)
    const int nb = static_cast<int>(p.H / 128);
    int64_t S = (4LL * dev.num_sms + p.T - 1) / p.T;
    if (S > nb) S = nb;
    if (S < 1) S = 1;
    int nbs = static_cast<int>((nb + S - 1) / S);
    if (nbs % 4 != 0 && nbs > 4 && nb % 4 == 0) nbs = (nbs + 3) / 4 * 4;
    S = (nb + nbs - 1) / nbs;
    if (S > 65535) return cudaErrorInvalidValue;
    const LLSmem L = ll_smem(nbs, p.E);
    if (L.total > dev.max_smem_optin) return cudaErrorInvalidValue;
    const bool peer = p.peer_recv_x != nullptr;
    err = cudaFuncSetAttribute(peer ? ll_dispatch_kernel<true> : ll_dispatch_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
    if (err != cudaSuccess) return err;
    const int pairs = (nbs + 1) / 2;
    int threads = 32 * (pairs < 2 ? 2 : pairs);
    if (threads > kLLMaxThreads) threads = kLLMaxThreads;
    // a plain launch: as a programmatic dependent it measured slower (4.73 -> 4.94 us per
    // call back to back), its 640 early CTAs competing with the previous kernel's
    const dim3 grid(static_cast<unsigned>(p.T), static_cast<unsigned>(S));
    if (peer)
        ll_dispatch_kernel<true><<<grid, threads, L.total, stream>>>(p, nbs);
    else
        ll_dispatch_kernel<false><<<grid, threads, L.total, stream>>>(p, nbs);
    return cudaGetLastError();
}

cudaError_t launch_wait_probe(uint32_t* status, uint32_t* flag, uint64_t timeout_ns,
                              cudaStream_t stream) {
    wait_probe_kernel<<<1, 1, 0, stream>>>(status, flag, timeout_ns);
    return cudaGetLastError();
}

}  // namespace ep
