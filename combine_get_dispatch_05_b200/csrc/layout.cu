// layout.cu -- routing layout of topk_idx: a stable counting sort of the (token, k)
// pairs by expert id.
//
// The receive buffer is expert-major (expert id ascending, then token, then k), so
// logical partition p -- experts [p*E/P, (p+1)*E/P) -- is one contiguous slice of
// rows.  Dispatch returns this layout as its handle and combine consumes it
// (deepseek.csdn.net/67bd3eb22e30c863900615cc, section "使用示例": dispatch returns
// recv_x, recv_topk_idx, recv_topk_weights, handle).
//
// One cooperative kernel; CTA c owns a contiguous chunk of tokens:
//   1. stage the chunk's expert ids in shared memory, histogram them (shared-memory
//      atomics: counts do not depend on order), flag the partitions each token
//      touches, publish the chunk's counts;
//   2. arrive at a grid barrier, and while the other chunks arrive
//   3. rank inside the chunk: each warp takes a contiguous run of (t, k) entries, 32
//      at a time; a 32-step shuffle loop ranks every pair among equal ids in the
//      batch, giving its rank within the run; the per-warp counts are scanned
//      across the warps;
//   4. wait at the barrier (bounded);
//   5. every CTA reads all chunks' counts, scans the totals into expert offsets and
//      adds the counts of earlier chunks: base[e] = first row of e in this chunk;
//   6. row = base[e] + rows of e in earlier warps of the chunk + rank within the run.
// Deterministic: nothing depends on the order atomics land in.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kLayoutThreads = 512;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr size_t kRankTableBytes = 32 * 1024;  // per-warp count table budget (shared memory)

struct LayoutArgs {
    const int64_t* topk_idx;
    int64_t T;
    int32_t K, E, P, epp;
    int32_t chunk_tokens;  // tokens per CTA, a multiple of 32
    int32_t round_warps;   // warps ranking, each a contiguous run (bounded by the table budget)
    int32_t flags_vec;     // is_token_in_partition is 8-byte aligned and P % 8 == 0
    // partition mode (deduplicated dispatch): the slots of a token are the P
    // partitions and the "ids" are partitions (K = E = P, epp = 1 below); the
    // routing is read as K_src ids per token among E_src experts, epp_src per partition
    int32_t by_partition;
    int32_t K_src, E_src, epp_src;
    int32_t parts;         // thread groups splitting the chunks in the cross-chunk sums
    int32_t* chunk_expert;     // [G][E]
    int32_t* chunk_partition;  // [G][P]
    uint8_t* is_token_in_partition;
    int32_t* num_tokens_per_expert;
    int32_t* num_tokens_per_partition;
    int32_t* expert_offset;
    int32_t* num_recv;
    int32_t* row_of;
    int32_t* src_of;
    unsigned long long* bar;  // grid-barrier word (8-byte aligned)
    uint32_t* status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ unsigned long long atom_add_release_gpu(unsigned long long* p,
                                                                   unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.add.release.gpu.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
    return old;
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Grid barrier of the (co-resident, cooperatively launched) grid, split into an
// arrive and a wait so that a CTA can do independent work in between.  One 64-bit
// word holds (generation << 32 | arrivals): each CTA adds 1 with release semantics
// (its writes before the arrive become visible); the last arrival adds 2^32 - G,
// which bumps the generation and resets the count in one step; the others poll
// with acquire loads until the generation changes, for at most timeout_ns.
// Thread 0 of each CTA calls both; the returned token is the generation to leave.
__device__ __forceinline__ unsigned long long grid_arrive(unsigned long long* word) {
    const unsigned long long old = atom_add_release_gpu(word, 1ull);
    if ((old & 0xFFFFFFFFull) == gridDim.x - 1)
        atom_add_release_gpu(word, (1ull << 32) - gridDim.x);
    return old >> 32;
}

__device__ __forceinline__ bool grid_wait(const unsigned long long* word, unsigned long long gen,
                                          uint64_t timeout_ns) {
    if ((ld_acquire_gpu(word) >> 32) != gen) return true;
    const uint64_t t0 = globaltimer_ns();
    while ((ld_acquire_gpu(word) >> 32) == gen) {
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
    return true;
}

// The low 8 bits of m as eight 0/1 bytes (bit i -> byte i).
__device__ __forceinline__ uint2 flag_bytes(uint64_t m) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lo |= static_cast<uint32_t>((m >> i) & 1u) << (8 * i);
        hi |= static_cast<uint32_t>((m >> (i + 4)) & 1u) << (8 * i);
    }
    return make_uint2(lo, hi);
}

__global__ void __launch_bounds__(kLayoutThreads, 1) layout_kernel(LayoutArgs a) {
    pdl_launch_dependents();  // the dispatch kernel may start loading x
    extern __shared__ __align__(16) int sm[];
    const int K = a.K, E = a.E, P = a.P, W = a.round_warps;
    const int Es = E + 1;  // padded row stride of the per-warp table (no bank conflicts)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int* ent = sm;                                // [chunk_tokens * K] ids, -1 = skip
    int* base = ent + a.chunk_tokens * K;         // [E] counts, then next row per expert
    int* wcnt = base + E;                         // [W][E + 1] per-warp counts / first rows
    int* part = wcnt + W * Es;                    // [2][parts][E] partial sums over chunks
    int* phist = part + 2 * a.parts * E;          // [P]
    int* part_of = phist + P + 32 + 4;            // [E] partition of each expert
    int* rir = part_of + E;                       // [chunk_tokens * K] rank within the run
    int* warp_sums = phist + P;                   // [32]
    int* flag = warp_sums + 32;                   // [1]

    const int64_t c = blockIdx.x;
    const int64_t t0 = c * a.chunk_tokens;
    const int64_t t1 = min(a.T, t0 + a.chunk_tokens);
    const int n = t1 > t0 ? static_cast<int>((t1 - t0) * K) : 0;

    for (int e = tid; e < E; e += blockDim.x) {
        base[e] = 0;
        part_of[e] = e / a.epp;
    }
    for (int p = tid; p < P; p += blockDim.x) phist[p] = 0;
    bool bad = false;
    if (!a.by_partition) {
        for (int j = tid; j < n; j += blockDim.x) {
            const int64_t e = a.topk_idx[t0 * K + j];
            const bool ok = e >= 0 && e < E;
            bad |= (e != -1) && !ok;
            ent[j] = ok ? static_cast<int>(e) : -1;
        }
    } else {
        // slot p of token t holds p if the token names any expert of partition p
        for (int tl = tid; tl < t1 - t0; tl += blockDim.x) {
            uint64_t mask = 0;
            for (int k = 0; k < a.K_src; ++k) {
                const int64_t e = a.topk_idx[(t0 + tl) * a.K_src + k];
                const bool ok = e >= 0 && e < a.E_src;
                bad |= (e != -1) && !ok;
                if (ok) mask |= 1ull << (e / a.epp_src);
            }
            for (int p = 0; p < K; ++p) ent[tl * K + p] = ((mask >> p) & 1u) ? p : -1;
        }
    }
    if (bad) raise_status(a.status, kDevIndexRange);
    __syncthreads();

    // 1. histogram and partition flags
    for (int j = tid; j < n; j += blockDim.x)
        if (ent[j] >= 0) atomicAdd(&base[ent[j]], 1);
    // token -> partition flags: every thread takes one token's K slots (K <= 32
    // consecutive ids in shared memory), ORs its partition bits, writes the P
    // flags; per-partition token counts by ballot
    for (int tb = warp * 32; tb < t1 - t0; tb += blockDim.x) {  // warp-uniform trip count
        const int tl = tb + lane;
        uint64_t mask = 0;
        if (tl < t1 - t0) {
#pragma unroll 4
            for (int k = 0; k < K; ++k) {
                const int e = ent[tl * K + ((k + lane) % K)];  // rotated: fewer bank conflicts
                if (e >= 0) mask |= 1ull << part_of[e];
            }
            uint8_t* flags = a.is_token_in_partition + (t0 + tl) * P;
            if (a.flags_vec) {
                for (int p = 0; p < P; p += 8)
                    *reinterpret_cast<uint2*>(flags + p) = flag_bytes(mask >> p);
            } else {
                for (int p = 0; p < P; ++p) flags[p] = static_cast<uint8_t>((mask >> p) & 1u);
            }
        }
        for (int p = 0; p < P; ++p) {
            const unsigned b = __ballot_sync(0xffffffffu, (mask >> p) & 1u);
            if (lane == 0 && b) atomicAdd(&phist[p], __popc(b));
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) a.chunk_expert[c * E + e] = base[e];
    for (int p = tid; p < P; p += blockDim.x) a.chunk_partition[c * P + p] = phist[p];

    // 2. publish: arrive at the grid barrier (release), but do not wait yet
    __syncthreads();
    unsigned long long gen = 0;
    if (tid == 0) gen = grid_arrive(a.bar);

    // 3. chunk-local ranks, which need no other chunk.  The n entries are split into
    //    W contiguous runs, one per warp, taken 32 at a time; a shuffle loop ranks
    //    equal ids inside a batch and a running per-warp count per expert turns that
    //    into the entry's rank within the run (kept in shared memory).  The per-warp
    //    counts are then scanned across the W warps: wcnt[w][e] = rows of e in this
    //    chunk before warp w's run.
    const int run = (n + W * 32 - 1) / (W * 32) * 32;  // entries per warp, multiple of 32
    for (int i = tid; i < W * Es; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    if (warp < W) {
        int* my = wcnt + warp * Es;
        const int j0 = warp * run, j1 = min(n, j0 + run);
        for (int j = j0 + lane; j - lane < j1; j += 32) {
            const bool in = j < j1;
            const int e = in ? ent[j] : -1;
            int rank = 0, same = 0;  // equal ids in lower lanes / in the whole batch
#pragma unroll
            for (int l = 0; l < 32; ++l) {
                const int el = __shfl_sync(0xffffffffu, e, l);
                same += el == e ? 1 : 0;
                rank += (l < lane && el == e) ? 1 : 0;
            }
            if (e >= 0) rir[j] = my[e] + rank;
            __syncwarp();
            if (e >= 0 && rank == 0) my[e] += same;  // first lane of its id
            __syncwarp();
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        int r = 0;
        for (int w = 0; w < W; ++w) {
            const int v = wcnt[w * Es + e];
            wcnt[w * Es + e] = r;
            r += v;
        }
    }

    // 4. wait for every chunk's counts
    if (tid == 0) *flag = grid_wait(a.bar, gen, a.timeout_ns) ? 1 : 0;
    __syncthreads();
    if (!*flag) {
        if (tid == 0) raise_status(a.status, kDevTimeout);
        return;
    }

    // 5. per expert: rows in all chunks and in earlier chunks.  `parts` groups of
    //    threads split the chunks; each thread issues its loads 16 at a time into
    //    registers so a whole batch is in flight (a loop over a runtime stride would
    //    wait for every load in turn).  CTA p < P also sums partition p's tokens.
    const int64_t G = gridDim.x;
    int ptot = 0;
    if (c < P && warp == (blockDim.x >> 5) - 1) {
        for (int64_t cc = lane; cc < G; cc += 32) ptot += __ldcg(a.chunk_partition + cc * P + c);
    }
    for (int i = tid; i < a.parts * E; i += blockDim.x) {
        const int e = i % E, q = i / E;
        int tot = 0, before = 0;
        for (int64_t c0 = q; c0 < G; c0 += 16 * static_cast<int64_t>(a.parts)) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int64_t cc = c0 + static_cast<int64_t>(u) * a.parts;
                v[u] = cc < G ? __ldcg(a.chunk_expert + cc * E + e) : 0;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int64_t cc = c0 + static_cast<int64_t>(u) * a.parts;
                tot += v[u];
                before += cc < c ? v[u] : 0;
            }
        }
        part[q * E + e] = tot;
        part[(a.parts + q) * E + e] = before;
    }
    if (c < P && warp == (blockDim.x >> 5) - 1) {
        ptot = __reduce_add_sync(0xffffffffu, ptot);
        if (lane == 0) a.num_tokens_per_partition[c] = ptot;
    }
    __syncthreads();
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        const int e = e0 + tid;
        int tot = 0, before = 0;
        if (e < E) {
            for (int q = 0; q < a.parts; ++q) {
                tot += part[q * E + e];
                before += part[(a.parts + q) * E + e];
            }
        }
        int tile_total;
        const int excl = block_exclusive_scan(tot, warp_sums, &tile_total);
        if (e < E) {
            base[e] = carry + excl + before;
            if (c == 0) {
                a.num_tokens_per_expert[e] = tot;
                a.expert_offset[e] = carry + excl;
            }
        }
        carry += tile_total;
    }
    if (c == 0 && tid == 0) {
        a.expert_offset[E] = carry;
        *a.num_recv = carry;
    }
    // partitions beyond the grid (P > G) hold the remaining sums
    for (int p = static_cast<int>(G) + static_cast<int>(c); p < P; p += static_cast<int>(G)) {
        if (warp == 0) {
            int t2 = 0;
            for (int64_t cc = lane; cc < G; cc += 32) t2 += __ldcg(a.chunk_partition + cc * P + p);
            t2 = __reduce_add_sync(0xffffffffu, t2);
            if (lane == 0) a.num_tokens_per_partition[p] = t2;
        }
    }
    __syncthreads();

    // 6. rows: first row of e in this chunk + rows before this warp's run + rank in run
    for (int j = tid; j < n; j += blockDim.x) {
        const int e = ent[j];
        const int row = e >= 0 ? base[e] + wcnt[(j / run) * Es + e] + rir[j] : -1;
        const int64_t g = t0 * K + j;
        a.row_of[g] = row;
        if (row >= 0) a.src_of[row] = static_cast<int32_t>(g);
    }
}

// Tokens per CTA: about kTargetChunk, but never more CTAs than SMs (the grid must
// be co-resident for its barrier).
constexpr int64_t kTargetChunk = 128;

int64_t layout_grid(int64_t T, int num_sms) {
    int64_t g = (T + kTargetChunk - 1) / kTargetChunk;
    if (g > num_sms) g = num_sms;
    return g < 1 ? 1 : g;
}

}  // namespace

int64_t max_layout_chunks(int64_t num_tokens) {
    const int64_t g = (num_tokens + kTargetChunk - 1) / kTargetChunk;
    return g < 1 ? 1 : g;
}

Workspace carve_workspace(void* ws, int64_t num_tokens, int32_t num_experts) {
    uint8_t* b = static_cast<uint8_t*>(ws);
    Workspace w;
    w.status = reinterpret_cast<uint32_t*>(b + kWsStatus);
    w.bar = reinterpret_cast<unsigned long long*>(b + kWsBar);
    w.probe_flag = reinterpret_cast<uint32_t*>(b + kWsProbeFlag);
    w.chunk_expert = reinterpret_cast<int32_t*>(b + kWsHeader);
    w.chunk_partition =
        w.chunk_expert + static_cast<int64_t>(num_experts) * max_layout_chunks(num_tokens);
    return w;
}

cudaError_t launch_layout(int64_t T, int32_t K, int32_t E, int32_t P, const int64_t* topk_idx,
                          const ep_layout& lay, const Workspace& ws, cudaStream_t stream,
                          bool by_partition) {
    const int32_t K_src = K, E_src = E, epp_src = E / P;
    if (by_partition) {  // slots and ids are partitions
        K = P;
        E = P;
    }
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const int64_t G = layout_grid(T, dev.num_sms);
    int64_t chunk = (T + G - 1) / G;
    chunk = (chunk + 31) / 32 * 32;
    if (chunk < 32) chunk = 32;
    int W = static_cast<int>(kRankTableBytes / (sizeof(int) * (static_cast<size_t>(E) + 1)));
    if (W > kLayoutWarps) W = kLayoutWarps;
    if (W < 1) W = 1;
    // thread groups splitting the chunks: enough that every thread has an
    // (expert, group) pair, at least one, at most one per chunk
    int parts = (kLayoutThreads + E - 1) / E;
    if (parts > G) parts = static_cast<int>(G);
    if (parts < 1) parts = 1;

    LayoutArgs a;
    a.topk_idx = topk_idx;
    a.T = T;
    a.K = K;
    a.E = E;
    a.P = P;
    a.epp = by_partition ? 1 : E / P;
    a.by_partition = by_partition ? 1 : 0;
    a.K_src = K_src;
    a.E_src = E_src;
    a.epp_src = epp_src;
    a.chunk_tokens = static_cast<int32_t>(chunk);
    a.round_warps = W;
    a.flags_vec = (P % 8 == 0) && ((reinterpret_cast<uintptr_t>(lay.is_token_in_partition) & 7u) == 0);
    a.parts = parts;
    a.chunk_expert = ws.chunk_expert;
    a.chunk_partition = ws.chunk_partition;
    a.is_token_in_partition = lay.is_token_in_partition;
    a.num_tokens_per_expert = lay.num_tokens_per_expert;
    a.num_tokens_per_partition = lay.num_tokens_per_partition;
    a.expert_offset = lay.expert_offset;
    a.num_recv = lay.num_recv;
    a.row_of = lay.row_of;
    a.src_of = lay.src_of;
    a.bar = ws.bar;
    a.status = ws.status;
    a.timeout_ns = kDefaultTimeoutNs;

    const size_t smem =
        sizeof(int) * (static_cast<size_t>(chunk) * K + static_cast<size_t>(E) +
                       static_cast<size_t>(W) * (E + 1) + 2 * static_cast<size_t>(parts) * E + P +
                       32 + 4 + static_cast<size_t>(E) + static_cast<size_t>(chunk) * K);
    if (smem > dev.max_smem_optin) return cudaErrorInvalidValue;
    err = cudaFuncSetAttribute(layout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    // First kernel of the call: an ordinary (not programmatic) launch, so it waits for
    // all earlier work in the stream.  Cooperative: the grid barrier needs every CTA
    // resident at once.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(G));
    cfg.blockDim = dim3(kLayoutThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, layout_kernel, a);
}

}  // namespace ep
