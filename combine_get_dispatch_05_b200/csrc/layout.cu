// layout.cu -- routing layout of topk_idx: a stable counting sort of the (token, k)
// pairs by expert id.
//
// The receive buffer is expert-major (expert id ascending, then token, then k), so
// logical partition p -- experts [p*E/P, (p+1)*E/P) -- is one contiguous slice of
// rows.  Dispatch returns this layout as its handle and combine consumes it
// (deepseek.csdn.net/67bd3eb22e30c863900615cc, section "使用示例": dispatch returns
// recv_x, recv_topk_idx, recv_topk_weights, handle).
//
// CTA c owns a contiguous chunk of tokens:
//   0. before waiting for the preceding kernel, prefetch the chunk's ids into L2;
//   1. load the chunk's expert ids into shared memory (many loads in flight per
//      thread), histogram them and OR each token's partition bits (shared-memory
//      atomics: neither depends on the order they land in);
//   2. write the token -> partition flags, count tokens per partition (ballots),
//      publish the chunk's counts and arrive at a barrier of all CTAs;
//   3. while the others arrive, rank inside the chunk: each warp takes a contiguous
//      run of (t, k) entries, 32 at a time; lanes with equal ids find each other
//      with one ballot per id bit, which gives every entry its rank within the run;
//      the per-warp counts are scanned across the warps;
//   4. wait at the barrier;
//   5. read all chunks' counts, scan the totals into expert offsets and add the
//      counts of earlier chunks: base[e] = first row of e in this chunk;
//   6. row = base[e] + rows of e in earlier warps of the chunk + rank within the run;
//      row_of is written in token order, src_of after sorting the chunk's rows in
//      shared memory, so that its stores go to contiguous rows.
// Deterministic: nothing depends on the order atomics land in.
//
// Two kernels share these phases:
//   * layout_single_kernel: one CTA for batches of up to 4096 (token, k) entries
//     (decode-sized); there is no other chunk, so no barrier and no exchange.
//   * layout_kernel: a cooperative grid of up to one CTA per SM.  Counts go through
//     a global table; the barrier is a bounded spin on one 64-bit word.  (A single
//     thread-block cluster exchanging counts through distributed shared memory was
//     measured slower than this grid on B200 for every multi-CTA batch tried.)
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kLayoutThreads = 512;
constexpr int kSingleThreads = 1024;
constexpr int64_t kSingleMaxEntries = 4096;     // batches the one-CTA kernel takes
constexpr size_t kRankTableBytes = 32 * 1024;    // per-warp count table budget (grid kernel)
constexpr size_t kSingleRankTableBytes = 40 * 1024;

struct LayoutArgs {
    const int64_t* topk_idx;
    int64_t T;
    int32_t K, E, P, epp;
    int32_t chunk_tokens;  // tokens per CTA, a multiple of 32
    int32_t round_warps;   // warps ranking, each a contiguous run (bounded by the table budget)
    int32_t id_bits;       // bits of an id in 0..E (E marks a skipped slot)
    int32_t flags_vec;     // is_token_in_partition is 8-byte aligned and P % 8 == 0
    int32_t sort_src;      // stage src_of in shared memory (room for it)
    // partition mode (deduplicated dispatch): the slots of a token are the P
    // partitions and the "ids" are partitions (K = E = P, epp = 1 below); the
    // routing is read as K_src ids per token among E_src experts, epp_src per partition
    int32_t by_partition;
    int32_t K_src, E_src, epp_src;
    int32_t parts;             // thread groups splitting the chunks in the cross-chunk sums
    int32_t* chunk_expert;     // [G][E] (grid kernel)
    int32_t* chunk_partition;  // [G][P] (grid kernel)
    uint8_t* is_token_in_partition;
    int32_t* num_tokens_per_expert;
    int32_t* num_tokens_per_partition;
    int32_t* expert_offset;
    int32_t* num_recv;
    int32_t* row_of;
    int32_t* src_of;
    unsigned long long* bar;  // grid-barrier word (8-byte aligned; grid kernel)
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

// L2 prefetch of the ids of tokens [t0, t1), issued before the kernel waits for its
// predecessor: a prefetch has no result, so it may run before the producer of
// topk_idx is done (that producer's stores reach L2, where the loads after the wait
// read), and it takes the ids' DRAM latency off the layout's critical path.
__device__ __forceinline__ void prefetch_ids(const LayoutArgs& a, int64_t t0, int64_t t1) {
    if (t1 <= t0) return;
    const int64_t per_tok = a.by_partition ? a.K_src : a.K;
    const char* src = reinterpret_cast<const char*>(a.topk_idx + t0 * per_tok);
    const int64_t bytes = (t1 - t0) * per_tok * 8;
    for (int64_t off = static_cast<int64_t>(threadIdx.x) * 128; off < bytes;
         off += static_cast<int64_t>(blockDim.x) * 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(src + off));
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

// Exclusive scan of two values over the CTA (one pair per thread); warp_sums holds
// 64 ints.  Returns the two exclusive prefixes and the two CTA totals.
__device__ __forceinline__ void block_scan2(int v0, int v1, int* warp_sums, int* x0, int* x1,
                                            int* tot0, int* tot1) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    int a = v0, b = v1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, a, o);
        const int yb = __shfl_up_sync(0xffffffffu, b, o);
        if (lane >= o) {
            a += ya;
            b += yb;
        }
    }
    if (lane == 31) {
        warp_sums[warp] = a;
        warp_sums[32 + warp] = b;
    }
    __syncthreads();
    if (warp == 0) {
        int wa = lane < nwarps ? warp_sums[lane] : 0;
        int wb = lane < nwarps ? warp_sums[32 + lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int ya = __shfl_up_sync(0xffffffffu, wa, o);
            const int yb = __shfl_up_sync(0xffffffffu, wb, o);
            if (lane >= o) {
                wa += ya;
                wb += yb;
            }
        }
        warp_sums[lane] = wa;  // inclusive over warps
        warp_sums[32 + lane] = wb;
    }
    __syncthreads();
    *x0 = (warp > 0 ? warp_sums[warp - 1] : 0) + a - v0;
    *x1 = (warp > 0 ? warp_sums[32 + warp - 1] : 0) + b - v1;
    *tot0 = warp_sums[nwarps - 1];
    *tot1 = warp_sums[32 + nwarps - 1];
    __syncthreads();  // warp_sums may be reused by the caller
}

// Shared memory of both kernels (int units unless noted):
//   tmask[chunk] (u64, partition bits per token) | ent[n] | rir[n] | srt[2n] (when
//   sort_src) | cnt[E] | base[E] | lofs[E] | part_of[E] | wcnt[W][E+1] | phist[P] |
//   warp_sums[64] | flag[4] | (grid kernel) part[2][parts][E]
struct Smem {
    unsigned long long* tmask;
    int* ent;
    int* rir;
    int* srt;
    int* cnt;
    int* base;
    int* lofs;
    int* part_of;
    int* wcnt;
    int* phist;
    int* warp_sums;
    int* flag;
    int* part;
};

size_t smem_ints(int64_t chunk, int K, int E, int P, int W, bool sort_src, int parts) {
    const size_t n = static_cast<size_t>(chunk) * K;
    return 2 * static_cast<size_t>(chunk) + (sort_src ? 4 : 2) * n + 4 * static_cast<size_t>(E) +
           static_cast<size_t>(W) * (E + 1) + P + 64 + 4 + 2 * static_cast<size_t>(parts) * E;
}

__device__ __forceinline__ Smem carve_smem(void* raw, const LayoutArgs& a) {
    Smem s;
    const int n = a.chunk_tokens * a.K;
    s.tmask = static_cast<unsigned long long*>(raw);
    s.ent = reinterpret_cast<int*>(s.tmask + a.chunk_tokens);
    s.rir = s.ent + n;
    s.srt = s.rir + n;
    s.cnt = s.srt + (a.sort_src ? 2 * n : 0);
    s.base = s.cnt + a.E;
    s.lofs = s.base + a.E;
    s.part_of = s.lofs + a.E;
    s.wcnt = s.part_of + a.E;
    s.phist = s.wcnt + a.round_warps * (a.E + 1);
    s.warp_sums = s.phist + a.P;
    s.flag = s.warp_sums + 64;
    s.part = s.flag + 4;
    return s;
}

// Phases 1-2: ids, histogram, partition bits, flags, per-partition token counts.
// Ends with the chunk's cnt[E] and phist[P] complete (after a __syncthreads).
__device__ __forceinline__ void count_chunk(const LayoutArgs& a, const Smem& s, int64_t t0,
                                            int64_t t1, int n) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = a.K, E = a.E, P = a.P;
    const int nt = static_cast<int>(t1 - t0);
    for (int e = tid; e < E; e += blockDim.x) {
        s.cnt[e] = 0;
        s.part_of[e] = e / a.epp;
    }
    for (int p = tid; p < P; p += blockDim.x) s.phist[p] = 0;
    for (int t = tid; t < nt; t += blockDim.x) s.tmask[t] = 0;
    __syncthreads();
    bool bad = false;
    if (!a.by_partition) {
        // 8 loads per thread in flight (a plain strided loop would wait for each)
        const int64_t* src = a.topk_idx + t0 * K;
        for (int j0 = tid; j0 < n; j0 += 8 * static_cast<int>(blockDim.x)) {
            int64_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u * static_cast<int>(blockDim.x);
                v[u] = j < n ? src[j] : -1;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u * static_cast<int>(blockDim.x);
                const bool ok = v[u] >= 0 && v[u] < E;
                bad |= (v[u] != -1) && !ok;
                if (j < n) {
                    const int e = ok ? static_cast<int>(v[u]) : -1;
                    s.ent[j] = e;
                    if (ok) {
                        atomicAdd(&s.cnt[e], 1);
                        atomicOr(&s.tmask[j / K], 1ull << s.part_of[e]);
                    }
                }
            }
        }
    } else {
        // slot p of token t holds p if the token names any expert of partition p
        for (int tl = tid; tl < nt; tl += blockDim.x) {
            uint64_t mask = 0;
#pragma unroll 8
            for (int k = 0; k < a.K_src; ++k) {
                const int64_t e = a.topk_idx[(t0 + tl) * a.K_src + k];
                const bool ok = e >= 0 && e < a.E_src;
                bad |= (e != -1) && !ok;
                if (ok) mask |= 1ull << (static_cast<int>(e) / a.epp_src);  // 32-bit division
            }
            s.tmask[tl] = mask;
            for (int p = 0; p < K; ++p) {
                const bool in = (mask >> p) & 1u;
                s.ent[tl * K + p] = in ? p : -1;
                if (in) atomicAdd(&s.cnt[p], 1);
            }
        }
    }
    if (bad) raise_status(a.status, kDevIndexRange);
    __syncthreads();
    // flags and per-partition token counts, one token per thread
    for (int tb = warp * 32; tb < nt; tb += blockDim.x) {  // warp-uniform trip count
        const int tl = tb + lane;
        const uint64_t mask = tl < nt ? s.tmask[tl] : 0;
        if (tl < nt) {
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
            if (lane == 0 && b) atomicAdd(&s.phist[p], __popc(b));
        }
    }
    __syncthreads();
}

// Phase 3: chunk-local ranks, which need no other chunk.  The n entries are split
// into W contiguous runs of `run` entries, one per warp, taken 32 at a time.  Lanes
// holding equal ids find each other with one ballot per id bit (skipped slots carry
// the id E); a running per-warp count per expert turns the rank among them into the
// entry's rank within the run (rir).  The per-warp counts are then scanned across the
// W warps: wcnt[w][e] = rows of e in this chunk before warp w's run.  Ends with a
// __syncthreads.
__device__ __forceinline__ void rank_chunk(const LayoutArgs& a, const Smem& s, int n, int run) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, W = a.round_warps, Es = E + 1;  // padded rows: no bank conflicts
    for (int i = tid; i < W * Es; i += blockDim.x) s.wcnt[i] = 0;
    __syncthreads();
    if (warp < W) {
        int* my = s.wcnt + warp * Es;
        const unsigned lower = (1u << lane) - 1u;
        const int j0 = warp * run, j1 = min(n, j0 + run);
        for (int j = j0 + lane; j - lane < j1; j += 32) {
            const int e = j < j1 ? s.ent[j] : -1;
            const unsigned key = e >= 0 ? static_cast<unsigned>(e) : static_cast<unsigned>(E);
            unsigned peers = 0xffffffffu;
            for (int b = 0; b < a.id_bits; ++b) {
                const unsigned bit = (key >> b) & 1u;
                const unsigned bal = __ballot_sync(0xffffffffu, bit);
                peers &= bit ? bal : ~bal;
            }
            const int rank = __popc(peers & lower);
            if (e >= 0) s.rir[j] = my[e] + rank;
            __syncwarp();
            if (e >= 0 && rank == 0) my[e] += __popc(peers);  // first lane of its id
            __syncwarp();
        }
    }
    __syncthreads();
    // scan over warps, 16 loads in flight per thread
    for (int e = tid; e < E; e += blockDim.x) {
        int r = 0;
        for (int w0 = 0; w0 < W; w0 += 16) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = w0 + u < W ? s.wcnt[(w0 + u) * Es + e] : 0;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (w0 + u < W) s.wcnt[(w0 + u) * Es + e] = r;
                r += v[u];
            }
        }
    }
    __syncthreads();
}

// Phase 5 (second half): given tot[e] (rows of e in all chunks) and before[e] (in
// earlier chunks) -- `get(e, &tot, &before)` supplies the pair -- scan the totals
// into expert offsets; base[e] = first row of e in this chunk, lofs[e] = first row
// of e among the chunk's own rows.  The writer CTA stores the per-expert outputs.
// Returns the number of the chunk's own rows.
template <class Get>
__device__ __forceinline__ int offsets_and_base(const LayoutArgs& a, const Smem& s, bool writer,
                                                Get get) {
    const int tid = threadIdx.x;
    int carry = 0, lcarry = 0;
    for (int e0 = 0; e0 < a.E; e0 += blockDim.x) {
        const int e = e0 + tid;
        int tot = 0, before = 0, mine = 0;
        if (e < a.E) {
            get(e, &tot, &before);
            mine = s.cnt[e];
        }
        int x0, x1, t0, t1;
        block_scan2(tot, mine, s.warp_sums, &x0, &x1, &t0, &t1);
        if (e < a.E) {
            s.base[e] = carry + x0 + before;
            s.lofs[e] = lcarry + x1;
            if (writer) {
                a.num_tokens_per_expert[e] = tot;
                a.expert_offset[e] = carry + x0;
            }
        }
        carry += t0;
        lcarry += t1;
    }
    if (writer && tid == 0) {
        a.expert_offset[a.E] = carry;
        *a.num_recv = carry;
    }
    return lcarry;
}

// Phase 6: row = first row of e in this chunk + rows before this warp's run + rank.
// row_of in token order; src_of either straight (scattered stores) or through the
// chunk's rows sorted in shared memory (stores to contiguous rows).
__device__ __forceinline__ void write_rows(const LayoutArgs& a, const Smem& s, int64_t t0, int n,
                                           int run, int nrows) {
    const int Es = a.E + 1;
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const int e = s.ent[j];
        const int64_t g = t0 * a.K + j;
        int row = -1;
        if (e >= 0) {
            const int local = s.wcnt[(j / run) * Es + e] + s.rir[j];
            row = s.base[e] + local;
            if (a.sort_src) {
                s.srt[2 * (s.lofs[e] + local)] = row;
                s.srt[2 * (s.lofs[e] + local) + 1] = static_cast<int32_t>(g);
            } else {
                a.src_of[row] = static_cast<int32_t>(g);
            }
        }
        a.row_of[g] = row;
    }
    if (a.sort_src) {
        __syncthreads();
        for (int r = threadIdx.x; r < nrows; r += blockDim.x) a.src_of[s.srt[2 * r]] = s.srt[2 * r + 1];
    }
}

__device__ __forceinline__ int run_length(int n, int W) {
    return (n + W * 32 - 1) / (W * 32) * 32;  // entries per warp, multiple of 32
}

// ---------------------------------------------------------- one-CTA kernel --

// The whole batch in one CTA: the chunk's counts are the totals.
__global__ void __launch_bounds__(kSingleThreads, 1) layout_single_kernel(LayoutArgs a) {
    prefetch_ids(a, 0, a.T);
    pdl_wait();               // the previous kernel (e.g. the one writing topk_idx) is complete
    pdl_launch_dependents();  // the dispatch kernel may start loading x
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const Smem s = carve_smem(smem_raw, a);
    const int64_t t1 = a.T;
    const int n = static_cast<int>(t1 * a.K);

    count_chunk(a, s, 0, t1, n);
    for (int p = threadIdx.x; p < a.P; p += blockDim.x) a.num_tokens_per_partition[p] = s.phist[p];
    const int run = run_length(n, a.round_warps);
    rank_chunk(a, s, n, run);
    const int nrows = offsets_and_base(a, s, true, [&](int e, int* tot, int* before) {
        *tot = s.cnt[e];
        *before = 0;
    });
    write_rows(a, s, 0, n, run, nrows);
}

// ------------------------------------------------------------ grid kernel --

__global__ void __launch_bounds__(kLayoutThreads, 1) layout_kernel(LayoutArgs a) {
    const int64_t c = blockIdx.x;
    const int64_t t0 = c * a.chunk_tokens;
    const int64_t t1 = min(a.T, t0 + a.chunk_tokens);
    prefetch_ids(a, t0, t1);
    pdl_wait();               // the previous kernel (e.g. the one writing topk_idx) is complete
    pdl_launch_dependents();  // the dispatch kernel may start loading x
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const Smem s = carve_smem(smem_raw, a);
    const int E = a.E, P = a.P;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int n = t1 > t0 ? static_cast<int>((t1 - t0) * a.K) : 0;

    count_chunk(a, s, t0, t1, n);
    for (int e = tid; e < E; e += blockDim.x) a.chunk_expert[c * E + e] = s.cnt[e];
    for (int p = tid; p < P; p += blockDim.x) a.chunk_partition[c * P + p] = s.phist[p];

    // publish: arrive at the grid barrier (release), but do not wait yet
    __syncthreads();
    unsigned long long gen = 0;
    if (tid == 0) gen = grid_arrive(a.bar);

    const int run = run_length(n, a.round_warps);
    rank_chunk(a, s, n, run);

    if (tid == 0) *s.flag = grid_wait(a.bar, gen, a.timeout_ns) ? 1 : 0;
    __syncthreads();
    if (!*s.flag) {
        if (tid == 0) raise_status(a.status, kDevTimeout);
        return;
    }

    // per expert: rows in all chunks and in earlier chunks.  `parts` groups of
    // threads split the chunks; each thread issues its loads 16 at a time into
    // registers so a whole batch is in flight (a loop over a runtime stride would
    // wait for every load in turn).  CTA p < P also sums partition p's tokens.
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
        s.part[q * E + e] = tot;
        s.part[(a.parts + q) * E + e] = before;
    }
    if (c < P && warp == (blockDim.x >> 5) - 1) {
        ptot = __reduce_add_sync(0xffffffffu, ptot);
        if (lane == 0) a.num_tokens_per_partition[c] = ptot;
    }
    __syncthreads();
    const int nrows = offsets_and_base(a, s, c == 0, [&](int e, int* tot, int* before) {
        int sum = 0, b = 0;
        for (int q = 0; q < a.parts; ++q) {
            sum += s.part[q * E + e];
            b += s.part[(a.parts + q) * E + e];
        }
        *tot = sum;
        *before = b;
    });
    // partitions beyond the grid (P > G) hold the remaining sums
    for (int p = static_cast<int>(G) + static_cast<int>(c); p < P; p += static_cast<int>(G)) {
        if (warp == 0) {
            int t2 = 0;
            for (int64_t cc = lane; cc < G; cc += 32) t2 += __ldcg(a.chunk_partition + cc * P + p);
            t2 = __reduce_add_sync(0xffffffffu, t2);
            if (lane == 0) a.num_tokens_per_partition[p] = t2;
        }
    }
    write_rows(a, s, t0, n, run, nrows);
}

// Tokens per CTA of the grid kernel: about kTargetChunk, but never more CTAs than
// SMs (the grid must be co-resident for its barrier).
constexpr int64_t kTargetChunk = 128;

int64_t layout_grid(int64_t T, int num_sms) {
    int64_t g = (T + kTargetChunk - 1) / kTargetChunk;
    if (g > num_sms) g = num_sms;
    return g < 1 ? 1 : g;
}

int rank_warps(size_t budget, int E, int max_warps) {
    int W = static_cast<int>(budget / (sizeof(int) * (static_cast<size_t>(E) + 1)));
    if (W > max_warps) W = max_warps;
    return W < 1 ? 1 : W;
}

int id_bits(int E) {  // bits of the ids 0..E
    int b = 1;
    while ((1 << b) <= E) ++b;
    return b;
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
    w.ticket = reinterpret_cast<int32_t*>(b + kWsTicket);
    w.done = reinterpret_cast<uint32_t*>(b + kWsDone);
    w.probe_flag = reinterpret_cast<uint32_t*>(b + kWsProbeFlag);
    w.chunk_expert = reinterpret_cast<int32_t*>(b + kWsHeader);
    w.chunk_partition =
        w.chunk_expert + static_cast<int64_t>(num_experts) * max_layout_chunks(num_tokens);
    return w;
}

cudaError_t layout_fits(int64_t T, int32_t K, int32_t E, int32_t P, bool by_partition,
                        bool* fits) {
    if (by_partition) {
        K = P;
        E = P;
    }
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    if (T * K <= kSingleMaxEntries) {
        const int W = rank_warps(kSingleRankTableBytes, E, kSingleThreads / 32);
        if (sizeof(int) * smem_ints(T > 0 ? T : 1, K, E, P, W, true, 0) <= dev.max_smem_optin) {
            *fits = true;
            return cudaSuccess;
        }
    }
    const int64_t G = layout_grid(T, dev.num_sms);
    int64_t chunk = (T + G - 1) / G;
    chunk = (chunk + 31) / 32 * 32;
    if (chunk < 32) chunk = 32;
    const int W = rank_warps(kRankTableBytes, E, kLayoutThreads / 32);
    int parts = (kLayoutThreads + E - 1) / E;
    if (parts > G) parts = static_cast<int>(G);
    if (parts < 1) parts = 1;
    *fits = sizeof(int) * smem_ints(chunk, K, E, P, W, false, parts) <= dev.max_smem_optin;
    return cudaSuccess;
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
    a.id_bits = id_bits(E);
    a.flags_vec = (P % 8 == 0) && ((reinterpret_cast<uintptr_t>(lay.is_token_in_partition) & 7u) == 0);
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

    // First kernel of the call: a programmatic dependent launch, so its CTAs may be
    // scheduled while the previous kernel in the stream finishes; each waits for it
    // (griddepcontrol.wait) before reading topk_idx.
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;

    // One CTA for small batches.
    const int64_t entries = T * K;
    if (entries <= kSingleMaxEntries) {
        const int64_t chunk = T > 0 ? T : 1;
        const int W = rank_warps(kSingleRankTableBytes, E, kSingleThreads / 32);
        const size_t smem = sizeof(int) * smem_ints(chunk, K, E, P, W, true, 0);
        if (smem <= dev.max_smem_optin) {
            a.chunk_tokens = static_cast<int32_t>(chunk);
            a.round_warps = W;
            a.sort_src = 1;
            a.parts = 0;
            err = cudaFuncSetAttribute(layout_single_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
            if (err != cudaSuccess) return err;
            cfg.gridDim = dim3(1);
            cfg.blockDim = dim3(kSingleThreads);
            cfg.dynamicSmemBytes = smem;
            return cudaLaunchKernelEx(&cfg, layout_single_kernel, a);
        }
    }

    // Otherwise the cooperative grid.
    const int64_t G = layout_grid(T, dev.num_sms);
    int64_t chunk = (T + G - 1) / G;
    chunk = (chunk + 31) / 32 * 32;
    if (chunk < 32) chunk = 32;
    const int W = rank_warps(kRankTableBytes, E, kLayoutThreads / 32);
    // thread groups splitting the chunks: enough that every thread has an
    // (expert, group) pair, at least one, at most one per chunk
    int parts = (kLayoutThreads + E - 1) / E;
    if (parts > G) parts = static_cast<int>(G);
    if (parts < 1) parts = 1;
    a.chunk_tokens = static_cast<int32_t>(chunk);
    a.round_warps = W;
    a.parts = parts;
    a.sort_src = sizeof(int) * smem_ints(chunk, K, E, P, W, true, parts) <= dev.max_smem_optin;
    const size_t smem = sizeof(int) * smem_ints(chunk, K, E, P, W, a.sort_src != 0, parts);
    if (smem > dev.max_smem_optin) return cudaErrorInvalidValue;
    err = cudaFuncSetAttribute(layout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    // Cooperative: the grid barrier needs every CTA resident at once.
    cfg.gridDim = dim3(static_cast<unsigned>(G));
    cfg.blockDim = dim3(kLayoutThreads);
    cfg.dynamicSmemBytes = smem;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, layout_kernel, a);
}

}  // namespace ep
