// layout.cu -- routing layout of topk_idx: a stable counting sort of the (token, k)
// pairs by expert id.
//
// The receive buffer is expert-major (expert id ascending, then token, then k), so
// logical partition p -- experts [p*E/P, (p+1)*E/P) -- is one contiguous slice of
// rows.  Dispatch returns this layout as its handle and combine consumes it
// (deepseek.csdn.net/67bd3eb22e30c863900615cc, section "使用示例": dispatch returns
// recv_x, recv_topk_idx, recv_topk_weights, handle).
//
// Two kernels, one CTA per chunk of kChunkTokens tokens:
//   count: per-chunk expert histogram (shared-memory atomics: counts do not depend
//          on order), token -> partition flags; the last CTA to finish (atomic
//          ticket, no waiting) scans the [expert][chunk] counts into expert offsets
//          and per-chunk row bases.
//   rank:  per warp, a match_any / popc rank of each pair among equal expert ids,
//          per-warp counts scanned across the CTA's warps, plus the chunk base:
//          row = expert_offset[e] + rows of e in earlier chunks
//                + rows of e in earlier warps of this chunk + rank in this warp.
//          Deterministic: the result never depends on the order atomics land in.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kCountThreads = 512;
constexpr int kRankThreads = kRankWarps * 32;

struct CountArgs {
    const int64_t* topk_idx;
    int64_t T;
    int32_t K, E, P, epp;
    int64_t Cs;  // chunk stride of the [E][Cs] / [P][Cs] arrays
    int32_t* chunk_expert;
    int32_t* chunk_partition;
    uint8_t* is_token_in_partition;
    int32_t* num_tokens_per_expert;
    int32_t* num_tokens_per_partition;
    int32_t* expert_offset;
    int32_t* num_recv;
    uint32_t* ticket;
    uint32_t* status;
};

__global__ void __launch_bounds__(kCountThreads) layout_count_kernel(CountArgs a) {
    pdl_launch_dependents();
    extern __shared__ __align__(16) int sm_count[];
    int* hist = sm_count;            // [E]
    int* phist = hist + a.E;         // [P]
    int* warp_sums = phist + a.P;    // [32]
    int* is_last = warp_sums + 32;   // [1]
    const int tid = threadIdx.x;

    for (int e = tid; e < a.E; e += blockDim.x) hist[e] = 0;
    for (int p = tid; p < a.P; p += blockDim.x) phist[p] = 0;
    __syncthreads();

    const int64_t c = blockIdx.x;
    const int64_t t0 = c * kChunkTokens;
    const int64_t t1 = min(a.T, t0 + kChunkTokens);
    bool bad = false;
    for (int64_t j = t0 * a.K + tid; j < t1 * a.K; j += blockDim.x) {
        const int64_t e = a.topk_idx[j];
        if (e == -1) continue;
        if (e < 0 || e >= a.E) {
            bad = true;
            continue;
        }
        atomicAdd(&hist[e], 1);
    }
    for (int64_t t = t0 + tid; t < t1; t += blockDim.x) {
        uint64_t mask = 0;
        for (int k = 0; k < a.K; ++k) {
            const int64_t e = a.topk_idx[t * a.K + k];
            if (e >= 0 && e < a.E) mask |= 1ull << (e / a.epp);
        }
        uint8_t* flags = a.is_token_in_partition + t * a.P;
        for (int p = 0; p < a.P; ++p) flags[p] = static_cast<uint8_t>((mask >> p) & 1u);
        while (mask) {
            const int p = __ffsll(static_cast<long long>(mask)) - 1;
            atomicAdd(&phist[p], 1);
            mask &= mask - 1;
        }
    }
    if (bad) raise_status(a.status, kDevIndexRange);
    __syncthreads();

    for (int e = tid; e < a.E; e += blockDim.x) a.chunk_expert[e * a.Cs + c] = hist[e];
    for (int p = tid; p < a.P; p += blockDim.x) a.chunk_partition[p * a.Cs + c] = phist[p];
    __threadfence();
    __syncthreads();
    if (tid == 0) *is_last = (atomicAdd(a.ticket, 1u) == gridDim.x - 1) ? 1 : 0;
    __syncthreads();
    if (!*is_last) return;

    // ---- last CTA: every other chunk's counts are published (fence before ticket) ----
    __threadfence();
    const int64_t C = gridDim.x;
    int carry = 0;
    for (int e0 = 0; e0 < a.E; e0 += blockDim.x) {
        const int e = e0 + tid;
        int tot = 0;
        if (e < a.E) {
            const int32_t* col = a.chunk_expert + e * a.Cs;
            int64_t cc = 0;
            for (; cc + 4 <= C; cc += 4) {
                const int4 v = __ldcg(reinterpret_cast<const int4*>(col + cc));
                tot += v.x + v.y + v.z + v.w;
            }
            for (; cc < C; ++cc) tot += __ldcg(col + cc);
        }
        int tile_total;
        const int excl = block_exclusive_scan(tot, warp_sums, &tile_total);
        if (e < a.E) {
            a.num_tokens_per_expert[e] = tot;
            a.expert_offset[e] = carry + excl;
            hist[e] = carry + excl;
        }
        carry += tile_total;
    }
    if (tid == 0) {
        a.expert_offset[a.E] = carry;
        *a.num_recv = carry;
    }
    __syncthreads();
    // chunk base of expert e = expert_offset[e] + rows of e in earlier chunks (in place)
    for (int e = tid; e < a.E; e += blockDim.x) {
        int32_t* col = a.chunk_expert + e * a.Cs;
        int run = hist[e];
        int64_t cc = 0;
        for (; cc + 4 <= C; cc += 4) {
            int4 v = __ldcg(reinterpret_cast<const int4*>(col + cc));
            int4 b;
            b.x = run; run += v.x;
            b.y = run; run += v.y;
            b.z = run; run += v.z;
            b.w = run; run += v.w;
            *reinterpret_cast<int4*>(col + cc) = b;
        }
        for (; cc < C; ++cc) {
            const int v = __ldcg(col + cc);
            col[cc] = run;
            run += v;
        }
    }
    for (int p = tid; p < a.P; p += blockDim.x) {
        const int32_t* col = a.chunk_partition + p * a.Cs;
        int tot = 0;
        for (int64_t cc = 0; cc < C; ++cc) tot += __ldcg(col + cc);
        a.num_tokens_per_partition[p] = tot;
    }
    if (tid == 0) *a.ticket = 0u;  // ready for the next launch on this workspace
}

struct RankArgs {
    const int64_t* topk_idx;
    int64_t T;
    int32_t K, E;
    int64_t Cs;
    const int32_t* chunk_base;  // [E][Cs], written by the count kernel's last CTA
    int32_t* row_of;
    int32_t* src_of;
};

__global__ void __launch_bounds__(kRankThreads) layout_rank_kernel(RankArgs a) {
    pdl_launch_dependents();
    extern __shared__ __align__(16) int sm_rank[];
    const int K = a.K, E = a.E;
    int* ent = sm_rank;                     // [kChunkTokens * K] expert ids, -1 = skip
    int* wcnt = ent + kChunkTokens * K;     // [kRankWarps][E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t c = blockIdx.x;
    const int64_t t0 = c * kChunkTokens;
    const int64_t t1 = min(a.T, t0 + kChunkTokens);
    const int n = static_cast<int>((t1 - t0) * K);

    // topk_idx is an input of the whole call, so it may be read before the count
    // kernel has finished.
    for (int j = tid; j < n; j += blockDim.x) {
        const int64_t e = a.topk_idx[t0 * K + j];
        ent[j] = (e >= 0 && e < E) ? static_cast<int>(e) : -1;
    }
    for (int i = tid; i < kRankWarps * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();

    // this warp's 32 tokens: entries [jw0, jw1)
    const int jw0 = min(n, warp * 32 * K);
    const int jw1 = min(n, jw0 + 32 * K);
    int* my = wcnt + warp * E;
    for (int j = jw0 + lane; j - lane < jw1; j += 32) {
        const int e = j < jw1 ? ent[j] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (__ffs(peers) - 1) == lane) my[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();

    pdl_wait();  // chunk bases are final
    for (int e = tid; e < E; e += blockDim.x) {
        int run = a.chunk_base[e * a.Cs + c];
        for (int w = 0; w < kRankWarps; ++w) {
            const int v = wcnt[w * E + e];
            wcnt[w * E + e] = run;
            run += v;
        }
    }
    __syncthreads();

    const unsigned lt = (1u << lane) - 1u;
    for (int j = jw0 + lane; j - lane < jw1; j += 32) {
        const bool in = j < jw1;
        const int e = in ? ent[j] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        int row = -1;
        if (e >= 0) row = my[e] + __popc(peers & lt);
        __syncwarp();
        if (e >= 0 && (__ffs(peers) - 1) == lane) my[e] += __popc(peers);
        __syncwarp();
        if (in) {
            const int64_t g = t0 * K + j;
            a.row_of[g] = row;
            if (row >= 0) a.src_of[row] = static_cast<int32_t>(g);
        }
    }
}

}  // namespace

int64_t num_chunks(int64_t num_tokens) { return (num_tokens + kChunkTokens - 1) / kChunkTokens; }

int64_t chunk_stride(int64_t num_tokens) {
    const int64_t c = num_chunks(num_tokens);
    return ((c > 0 ? c : 1) + 3) / 4 * 4;
}

Workspace carve_workspace(void* ws, int64_t num_tokens, int32_t num_experts) {
    uint8_t* base = static_cast<uint8_t*>(ws);
    Workspace w;
    w.status = reinterpret_cast<uint32_t*>(base + kWsStatus);
    w.ticket = reinterpret_cast<uint32_t*>(base + kWsTicket);
    w.probe_flag = reinterpret_cast<uint32_t*>(base + kWsProbeFlag);
    w.chunk_expert = reinterpret_cast<int32_t*>(base + kWsHeader);
    w.chunk_partition = w.chunk_expert + static_cast<int64_t>(num_experts) * chunk_stride(num_tokens);
    return w;
}

cudaError_t launch_layout(int64_t T, int32_t K, int32_t E, int32_t P, const int64_t* topk_idx,
                          const ep_layout& lay, const Workspace& ws, cudaStream_t stream) {
    const int64_t C = num_chunks(T);
    const int64_t Cs = chunk_stride(T);

    CountArgs ca;
    ca.topk_idx = topk_idx;
    ca.T = T;
    ca.K = K;
    ca.E = E;
    ca.P = P;
    ca.epp = E / P;
    ca.Cs = Cs;
    ca.chunk_expert = ws.chunk_expert;
    ca.chunk_partition = ws.chunk_partition;
    ca.is_token_in_partition = lay.is_token_in_partition;
    ca.num_tokens_per_expert = lay.num_tokens_per_expert;
    ca.num_tokens_per_partition = lay.num_tokens_per_partition;
    ca.expert_offset = lay.expert_offset;
    ca.num_recv = lay.num_recv;
    ca.ticket = ws.ticket;
    ca.status = ws.status;
    const size_t count_smem = sizeof(int) * (static_cast<size_t>(E) + P + 32 + 4);
    if (count_smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(
            layout_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)count_smem);
        if (err != cudaSuccess) return err;
    }
    // First kernel of the call: ordinary launch, so it waits for all earlier work.
    layout_count_kernel<<<dim3(static_cast<unsigned>(C > 0 ? C : 1)), kCountThreads, count_smem,
                          stream>>>(ca);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || C == 0) return err;

    RankArgs ra;
    ra.topk_idx = topk_idx;
    ra.T = T;
    ra.K = K;
    ra.E = E;
    ra.Cs = Cs;
    ra.chunk_base = ws.chunk_expert;
    ra.row_of = lay.row_of;
    ra.src_of = lay.src_of;
    const size_t rank_smem =
        sizeof(int) * (static_cast<size_t>(kChunkTokens) * K + static_cast<size_t>(kRankWarps) * E);
    if (rank_smem > 48 * 1024) {
        err = cudaFuncSetAttribute(layout_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)rank_smem);
        if (err != cudaSuccess) return err;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(C));
    cfg.blockDim = dim3(kRankThreads);
    cfg.dynamicSmemBytes = rank_smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, layout_rank_kernel, ra);
}

}  // namespace ep
