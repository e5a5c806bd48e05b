// dispatch.cu -- write every token to each of its receive rows.
//
// FP8 path ("DeepSeek 开源周第二弹：DeepEP", sections "DeepEP 的核心功能" (native FP8)
// and "DeepEP 的常规内核和低延迟内核" (FP8 dispatch)): per token, per 128-channel
// block, amax -> scale s = max(amax, 1e-4) / 448 -> q = e4m3_rne_satfinite(x / s);
// the E4M3 row and its fp32 scales go to every row_of[t, k].
//
// BF16 path: the row is copied bit for bit.
//
// Both kernels are persistent pipelines; a CTA takes its next token from a ticket
// counter in the workspace (one atomic per token), so CTAs that started late (on
// the SMs the layout kernel held) or that see less bandwidth take fewer tokens
// and all finish together.  The last CTA to finish re-zeroes the counter for the
// next call.  Which CTA writes a token does not change what is written: the
// output is deterministic.  Input rows arrive by 1-D bulk async copies
// (cp.async.bulk, mbarrier completion) into a ring of shared-memory stages, so
// several 14 KB rows per SM are in flight from HBM at once; output rows leave by
// bulk stores from shared memory, one per destination row, issued by one lane
// per top-k slot.  A token is read from HBM once and written K times: the
// traffic is the algorithmic minimum.  The x loads of the first stages are
// issued before waiting on the layout kernels (x is an input of the call), so
// they overlap the layout.
//
// Peer mode (template parameter kPeer; partitions are the ranks of a node): the
// storer lane of each row resolves the owner rank and the row there (peer_dest)
// and its bulk stores go to that rank's IPC-mapped receive buffer; everything
// else is the one-GPU pipeline.
#include "ep_device.cuh"
#include "ep_internal.h"
#include "ep_quant.cuh"

namespace ep {

namespace {

constexpr int kFp8InStages = 4;      // input ring: rows in flight from HBM per CTA
constexpr int kFp8MaxOutStages = 40;  // quantised rows staged per CTA, at most
constexpr int kFp8CtasPerSm = 2;      // the output ring fills this share of an SM
constexpr int kFp8MaxQuantWarps = 14; // quantiser warps per CTA, at most
constexpr int kFp8MaxStorers = 2;     // storer warps per CTA (taking alternate steps), at most
constexpr int kBf16Stages = 4;        // BF16 rows in flight per CTA
// Token log: the token of pipeline step i sits in tok[i % kTokLog] from the
// loader's ticket until the step's storer has read it; the storer then marks the
// entry consumed (kTokFree).  The loader runs at most (input stages + output stages
// + storers) steps ahead of the storers.  A storer peeks at the entry of its next
// step to prefetch that token's routing: a value >= 0 there can only be that
// step's token.
constexpr int kTokFree = -2;
constexpr int kTokLog = 64;
static_assert(kTokLog > kFp8InStages + kFp8MaxOutStages + kFp8MaxStorers, "token log too short");
static_assert(kTokLog > kBf16Stages + 1, "token log too short");
static_assert((kTokLog & (kTokLog - 1)) == 0, "token log size is a power of two");

// FP8 kernel shared memory: input ring | output ring (E4M3 row + scales per stage) |
// mbarriers | staged rows per output stage | token log | abort flag.
struct Fp8Smem {
    uint32_t in_bytes, q_bytes, s_bytes, out_bytes;
    uint32_t off_out, off_bars, off_rows, off_tok, off_flag, total;
};

__host__ __device__ inline Fp8Smem fp8_smem(int64_t H, int in_stages, int out_stages) {
    Fp8Smem s;
    const uint32_t nb = static_cast<uint32_t>(H / 128);
    s.in_bytes = static_cast<uint32_t>(H) * 2u;
    s.q_bytes = static_cast<uint32_t>(H);
    s.s_bytes = (nb * 4u + 15u) & ~15u;
    s.out_bytes = s.q_bytes + s.s_bytes;
    s.off_out = in_stages * s.in_bytes;
    s.off_bars = s.off_out + out_stages * s.out_bytes;
    s.off_rows = s.off_bars + 8u * 2u * (in_stages + out_stages);
    s.off_tok = s.off_rows + 4u * 32u * out_stages;
    s.off_flag = s.off_tok + 4u * kTokLog;
    s.total = s.off_flag + 16u;
    return s;
}

// A ring position: stage index and the parity of that stage's current use.
struct Ring {
    int stage = 0;
    uint32_t parity = 0;
    __device__ __forceinline__ void next(int n) {
        if (++stage == n) {
            stage = 0;
            parity ^= 1u;
        }
    }
};

// One token's routing as the storer lanes hold it: lane s the row of slot s,
// lane k routing entry k (id and weight).
struct Routing {
    int token = -1;
    int row = -1;
    int64_t e = -1;
    float wt = 0.0f;
};

__device__ __forceinline__ Routing load_routing(const DispatchParams& p, int t, int lane) {
    Routing r;
    r.token = t;
    if (lane < p.slots) r.row = p.row_of[static_cast<int64_t>(t) * p.slots + lane];
    if (lane < p.K) {
        r.e = p.topk_idx[static_cast<int64_t>(t) * p.K + lane];
        r.wt = p.topk_weights[static_cast<int64_t>(t) * p.K + lane];
    }
    return r;
}

// Prefetch for a token log entry read without waiting: only a real token (>= 0)
// is loaded; a free entry or the end marker gives an empty Routing.
__device__ __forceinline__ Routing peek_routing(const DispatchParams& p, int t, int lane) {
    return t >= 0 ? load_routing(p, t, lane) : Routing();
}

// Next token for this CTA, or -1 when the batch is exhausted.
__device__ __forceinline__ int take_ticket(const DispatchParams& p) {
    const int t = atomicAdd(p.ticket, 1);
    return t < p.T ? t : -1;
}

// Called by thread 0 after the whole CTA is done (every ticket it will take is
// taken): count the finished CTAs; the last one re-zeroes the ticket counter.
__device__ __forceinline__ void finish_tickets(const DispatchParams& p) {
    __threadfence();
    if (atomicAdd(p.done, 1u) == gridDim.x - 1) {
        atomicExch(p.ticket, 0);
        atomicExch(p.done, 0u);
    }
}

// Wait for a phase, giving up after timeout_ns or as soon as another warp of the
// CTA has given up (*abort_flag set).  On its own timeout it sets *abort_flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                              volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > timeout_ns) {
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// Where a storer lane writes its row: payload, scales, local id and weight arrays.
struct Dest {
    uint8_t* x;
    float* s;
    int32_t* i;
    float* w;
};

// Peer mode (partitions are ranks): slot k's row goes to the rank that owns its
// expert, at row_of[t, k] + peer_offset[e] there (lane k < K holds both the row
// and the id of slot k).  Deduplicated rows: lane q's row goes to rank q, at
// row_of[t, q] + peer_offset[q].  A row outside the owner's buffers (the owner
// receives more rows than it has room for) is dropped and reported.
__device__ __forceinline__ int peer_dest(const DispatchParams& p, int lane, int row, int64_t e,
                                         Dest& d) {
    if (row < 0) return -1;
    int part, at;
    if (p.dedup) {
        part = lane;
        at = lane;
    } else {
        if (e < 0 || e >= p.num_experts) {  // a handle that does not match topk_idx
            raise_status(p.status, kDevIndexRange);
            return -1;
        }
        at = static_cast<int>(e);
        part = at / p.experts_per_partition;
    }
    const int64_t r = static_cast<int64_t>(row) + p.peer_offset[at];
    if (r < 0 || r >= p.peer_rows) {
        raise_status(p.status, kDevCapacity);
        return -1;
    }
    d.x = static_cast<uint8_t*>(p.peer_recv_x[part]);
    d.s = p.peer_recv_scales ? p.peer_recv_scales[part] : nullptr;
    d.i = p.peer_recv_topk_idx[part];
    d.w = p.peer_recv_topk_weights[part];
    return static_cast<int>(r);
}

// Storer warps of the FP8 kernel.  Issuing a bulk store holds its warp for a few
// hundred ns, so at about 4 rows per token (deduplicated rows) one warp's issue time
// per token, not HBM, bounded a single storer (1.0 us of ~2 us per token); two
// storers issue in parallel (deduplicated normal workload 45.1 -> 41.0 us).  At 8
// rows per token the kernel is HBM-bound and a second storer only interleaves two
// tokens' row stores (in the step 60.6 -> 63.5 us): one storer.
inline int fp8_storers(const DispatchParams& p) { return p.dedup ? 2 : 1; }

// Metadata of one token's receive rows, written by the storer warp.  Per-expert
// rows: lane k owns slot k and writes the local id and weight of its row into
// ri / rw (its own destination's arrays in peer mode).
// Deduplicated rows (one per partition): lane p owns partition p's row and writes
// its K-entry lists into ri / rw, reading every slot's id and weight from the id
// lanes by shuffle (all lanes take part in the shuffles).
template <bool kPeer>
__device__ __forceinline__ void write_row_metadata(const DispatchParams& p, int lane, int row,
                                                   int64_t e, float wt, int32_t* ri, float* rw) {
    // lane k < K: partition and partition-local id of routing entry k, one 32-bit
    // division per lane (-1: not a valid expert id)
    const int epp = p.experts_per_partition;
    const bool valid = e >= 0 && e < p.num_experts;
    const int ei = valid ? static_cast<int>(e) : 0;
    const int part = valid ? ei / epp : -1;
    const int local = ei - (valid ? part : 0) * epp;
    if (!p.dedup) {
        if (lane < p.slots && row >= 0) {  // a row exists only for a valid id
            ri[row] = local;
            rw[row] = wt;
        }
        return;
    }
    for (int k = 0; k < p.K; ++k) {
        const int pk = __shfl_sync(0xffffffffu, part, k);
        const int lk = __shfl_sync(0xffffffffu, local, k);
        const float wk = __shfl_sync(0xffffffffu, wt, k);
        if (lane < p.slots && row >= 0) {
            const bool in = pk == lane;
            int32_t* li = kPeer ? ri : p.recv_topk_idx;
            float* lw = kPeer ? rw : p.recv_topk_weights;
            li[static_cast<int64_t>(row) * p.K + k] = in ? lk : -1;
            lw[static_cast<int64_t>(row) * p.K + k] = in ? wk : 0.0f;
        }
    }
}

// Warp-specialised pipeline, one CTA = 1 loader warp + nq quantiser warps + kNs storer
// warps, coupled only by mbarriers (no CTA-wide barrier between set-up and the end):
//   loader (warp 0, lane 0): takes a ticket, records the token in the token log and
//       bulk-loads its row into the input ring (in_full[s]: transaction bytes;
//       waits in_empty[s] before reusing a stage); when the tickets run out it
//       records -1 for one step per storer and arrives on in_full[s] without loads;
//   quantisers (warps 1..nq): quantise their share of the row's 128-channel blocks
//       from input stage s into output stage o, then arrive on in_empty[s] and
//       out_full[o] (waiting out_empty[o] before reusing an output stage); a -1
//       token is passed on without work, and the last one ends the warp;
//   storers (the last kNs warps, storer s taking steps s, s + kNs, ...): lane k
//       bulk-stores the staged row and its scales to row row_of[t, k], writes
//       recv_topk_idx / recv_topk_weights, and releases the output stage of its
//       previous step (out_empty) once those stores have read it; a -1 token ends
//       it.
// Only the storer reads what the layout kernel wrote, so only it waits on the
// programmatic dependency; loads and quantisation overlap the layout.
// kPeer: rows go to the owner ranks' buffers (peer_dest).
template <bool kPeer, int kNs>
__global__ void __launch_bounds__(32 * (kFp8MaxQuantWarps + 1 + kNs), kFp8CtasPerSm)
    dispatch_fp8_kernel(DispatchParams p) {
    static_assert(kNs >= 1 && kNs <= kFp8MaxStorers, "storer warps");
    pdl_launch_dependents();  // the next kernel (e.g. the combine) may be scheduled
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int ns = kNs;
    const int nq = (blockDim.x >> 5) - 1 - ns;
    const int64_t H = p.H;
    const int nb = static_cast<int>(H >> 7);
    const int NI = p.in_stages, NO = p.out_stages;
    const Fp8Smem L = fp8_smem(H, NI, NO);
    uint64_t* in_full = reinterpret_cast<uint64_t*>(sm + L.off_bars);
    uint64_t* in_empty = in_full + NI;
    uint64_t* out_full = in_empty + NI;
    uint64_t* out_empty = out_full + NO;
    int* rows_sm = reinterpret_cast<int*>(sm + L.off_rows);
    volatile int* tok = reinterpret_cast<volatile int*>(sm + L.off_tok);
    volatile int* abort_flag = reinterpret_cast<int*>(sm + L.off_flag);
    // row-major scales whose row is a whole number of 16-byte units go out with the
    // row's bulk store; otherwise (and block-major) the storer writes them one by one
    const bool scale_bulk = !p.scales_mn && (static_cast<uint32_t>(nb) * 4u) == L.s_bytes;

    if (tid == 0) {
        for (int s = 0; s < NI; ++s) {
            mbar_init(&in_full[s], 1);
            mbar_init(&in_empty[s], nq);
        }
        for (int o = 0; o < NO; ++o) {
            mbar_init(&out_full[o], nq);
            mbar_init(&out_empty[o], 1);
        }
        for (int j = 0; j < kTokLog; ++j) tok[j] = kTokFree;
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- loader
        if (lane == 0) {
            const uint8_t* x = static_cast<const uint8_t*>(p.x);
            int issued = 0;  // bulk loads issued (steps 0 .. issued-1)
            int ends = 0;    // end markers recorded
            Ring in;
            for (int i = 0;; ++i, in.next(NI)) {
                // the ticket's round trip overlaps the wait for a free stage
                const int t = (ns > 1 && ends) ? -1 : take_ticket(p);
                if (i >= NI && !wait_or_abort(&in_empty[in.stage], in.parity ^ 1u, p.timeout_ns,
                                              abort_flag))
                    break;
                tok[i & (kTokLog - 1)] = t;
                if (t < 0) {
                    mbar_arrive(&in_full[in.stage]);  // an end marker: no load
                    if (ns == 1 || ++ends == ns) break;
                    continue;
                }
                mbar_arrive_expect_tx(&in_full[in.stage], L.in_bytes);
                bulk_load(sm + in.stage * L.in_bytes, x + static_cast<int64_t>(t) * H * 2, L.in_bytes,
                          &in_full[in.stage]);
                ++issued;
            }
            if (*abort_flag) {
                // let this CTA's loads still in flight land before it exits: the
                // latest load of each stage is its barrier's current phase
                for (int j = issued - 1; j >= 0 && j >= issued - NI; --j)
                    mbar_wait_bounded(&in_full[j % NI], static_cast<uint32_t>((j / NI) & 1),
                                      kDefaultTimeoutNs);
            }
        }
    } else if (warp <= nq) {
        // ------------------------------------------------------------ quantisers
        const int qw = warp - 1;
        int ends = 0;
        Ring in, out;
        for (int i = 0;; ++i, in.next(NI), out.next(NO)) {
            if (!wait_or_abort(&in_full[in.stage], in.parity, p.timeout_ns, abort_flag)) break;
            if (i >= NO &&
                !wait_or_abort(&out_empty[out.stage], out.parity ^ 1u, p.timeout_ns, abort_flag))
                break;
            const int t = tok[i & (kTokLog - 1)];
            if (t >= 0) {
                uint8_t* out_q = sm + L.off_out + out.stage * L.out_bytes;
                quantize_row_fp8(sm + in.stage * L.in_bytes, out_q,
                                 reinterpret_cast<float*>(out_q + L.q_bytes), nb, qw, nq, lane,
                                 p.pow2_scales != 0);
                fence_proxy_async_smem();  // staged row visible to the bulk stores
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&in_empty[in.stage]);
                mbar_arrive(&out_full[out.stage]);
            }
            if (t < 0 && (ns == 1 || ++ends == ns)) break;
        }
    } else {
        // --------------------------------------------------------------- storers
        pdl_wait();  // row_of from the layout kernel is complete and visible
        uint8_t* recv_x = static_cast<uint8_t*>(p.recv_x);
        const int S = p.slots;
        const bool slot_lane = lane < S;  // lane s stores slot s's row
        int prev = -1;  // output stage of this warp's previous step
        Routing next;   // prefetched routing of this warp's next step's token
        Ring out;
        const int first = ns == 1 ? 0 : warp - 1 - nq;
        for (int j = 0; j < first; ++j) out.next(NO);
        for (int i = first;; i += ns) {
            const int o = out.stage;
            if (!wait_or_abort(&out_full[o], out.parity, p.timeout_ns, abort_flag)) break;
            const int t = tok[i & (kTokLog - 1)];
            if (t < 0) {
                if constexpr (ns > 1) {
                    // release the previous stage: the quantisers' last end marker may
                    // be waiting for it (a ring of at least three stages)
                    if (slot_lane) bulk_wait_read<0>();
                    __syncwarp();
                    if (lane == 0 && prev >= 0) mbar_arrive(&out_empty[prev]);
                }
                break;
            }
            const Routing cur = next.token == t ? next : load_routing(p, t, lane);
            __syncwarp();
            if (lane == 0) tok[i & (kTokLog - 1)] = kTokFree;
            next = peek_routing(p, tok[(i + ns) & (kTokLog - 1)], lane);
            int row = cur.row;
            const int64_t e = cur.e;
            const float wt = cur.wt;
            Dest d{recv_x, p.recv_scales, p.recv_topk_idx, p.recv_topk_weights};
            if constexpr (kPeer) row = peer_dest(p, lane, row, e, d);
            uint8_t* out_q = sm + L.off_out + o * L.out_bytes;
            const float* out_s = reinterpret_cast<const float*>(out_q + L.q_bytes);
            if (slot_lane) {
                if (row >= 0) {
                    bulk_store(d.x + static_cast<int64_t>(row) * H, out_q, L.q_bytes);
                    if (scale_bulk)
                        bulk_store(d.s + static_cast<int64_t>(row) * nb, out_s,
                                   static_cast<uint32_t>(nb) * 4u);
                }
                bulk_commit();
                rows_sm[o * 32 + lane] = row;
            }
            write_row_metadata<kPeer>(p, lane, row, e, wt, d.i, d.w);
            if constexpr (kPeer) {
                if (!scale_bulk && slot_lane && row >= 0)  // row-major: the lane's own row
                    for (int b = 0; b < nb; ++b) d.s[static_cast<int64_t>(row) * nb + b] = out_s[b];
            } else if (!scale_bulk) {
                __syncwarp();
                for (int idx = lane; idx < S * nb; idx += 32) {
                    const int k = idx / nb, b = idx - k * nb;
                    const int r = rows_sm[o * 32 + k];
                    if (r >= 0) {
                        const int64_t at = p.scales_mn ? b * p.scales_ld + r
                                                       : static_cast<int64_t>(r) * nb + b;
                        p.recv_scales[at] = out_s[b];
                    }
                }
            }
            // release the previous output stage once this warp's stores have read it
            if (slot_lane) bulk_wait_read<1>();
            __syncwarp();
            if (lane == 0 && prev >= 0) mbar_arrive(&out_empty[prev]);
            prev = o;
#pragma unroll
            for (int j = 0; j < ns; ++j) out.next(NO);
        }
        // the CTA may exit once its stores have read their stages; the grid completes
        // only when the writes have landed
        if (slot_lane) bulk_wait_read<0>();
    }
    __syncthreads();
    if (tid == 0) {
        if (*abort_flag) raise_status(p.status, kDevTimeout);
        finish_tickets(p);
    }
}

// BF16 rows are copied bit for bit, so the row staged by the bulk load is itself
// the source of the K bulk stores.  One CTA = a loader warp and a storer warp
// coupled by full/empty mbarriers over a ring of kBf16Stages rows:
//   loader (warp 0, lane 0): waits empty[s], takes a ticket, records the token in
//       the token log and bulk-loads its row into stage s (full[s] counts its
//       transaction bytes); when the tickets run out it records -1 and arrives on
//       full[s] without a load;
//   storer (warp 1): waits for the layout, then per step waits full[s], lane k
//       bulk-stores the row to row_of[t, k] and writes recv_topk_idx / weights;
//       once this token's stores have read the stage it arrives on empty[s].
// kPeer: rows go to the owner ranks' buffers (peer_dest).
template <bool kPeer>
__global__ void __launch_bounds__(64) dispatch_bf16_kernel(DispatchParams p) {
    pdl_launch_dependents();  // the next kernel (e.g. the combine) may be scheduled
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t H = p.H;
    const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kBf16Stages * row_bytes);
    uint64_t* empty = full + kBf16Stages;
    volatile int* tok = reinterpret_cast<volatile int*>(empty + kBf16Stages);
    volatile int* abort_flag = tok + kTokLog;

    if (tid == 0) {
        for (int s = 0; s < kBf16Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < kTokLog; ++j) tok[j] = kTokFree;
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- loader
        if (lane == 0) {
            const uint8_t* x = static_cast<const uint8_t*>(p.x);
            int64_t issued = 0;
            for (int64_t i = 0;; ++i) {
                const int s = static_cast<int>(i % kBf16Stages);
                const int t = take_ticket(p);  // overlaps the wait for a free stage
                if (i >= kBf16Stages &&
                    !wait_or_abort(&empty[s], static_cast<uint32_t>((i / kBf16Stages - 1) & 1),
                                   p.timeout_ns, abort_flag))
                    break;
                tok[i % kTokLog] = t;
                if (t < 0) {
                    mbar_arrive(&full[s]);  // the end marker: no load
                    break;
                }
                mbar_arrive_expect_tx(&full[s], row_bytes);
                bulk_load(sm + s * row_bytes, x + static_cast<int64_t>(t) * row_bytes, row_bytes,
                          &full[s]);
                ++issued;
            }
            if (*abort_flag) {
                for (int64_t j = issued - 1; j >= 0 && j >= issued - kBf16Stages; --j)
                    mbar_wait_bounded(&full[j % kBf16Stages],
                                      static_cast<uint32_t>((j / kBf16Stages) & 1),
                                      kDefaultTimeoutNs);
            }
        }
    } else {
        // ---------------------------------------------------------------- storer
        pdl_wait();  // row_of from the layout kernel is complete and visible
        uint8_t* recv_x = static_cast<uint8_t*>(p.recv_x);
        const int S = p.slots;
        const bool slot_lane = lane < S;  // lane s stores slot s's row
        Routing next;  // prefetched routing of the next step's token
        for (int64_t i = 0;; ++i) {
            const int s = static_cast<int>(i % kBf16Stages);
            if (!wait_or_abort(&full[s], static_cast<uint32_t>((i / kBf16Stages) & 1), p.timeout_ns,
                               abort_flag))
                break;
            const int t = tok[i % kTokLog];
            if (t < 0) break;
            const Routing cur = next.token == t ? next : load_routing(p, t, lane);
            __syncwarp();
            if (lane == 0) tok[i % kTokLog] = kTokFree;
            next = peek_routing(p, tok[(i + 1) % kTokLog], lane);
            int row = cur.row;
            const int64_t e = cur.e;
            const float wt = cur.wt;
            Dest d{recv_x, nullptr, p.recv_topk_idx, p.recv_topk_weights};
            if constexpr (kPeer) row = peer_dest(p, lane, row, e, d);
            if (slot_lane) {
                if (row >= 0)
                    bulk_store(d.x + static_cast<int64_t>(row) * row_bytes, sm + s * row_bytes,
                               row_bytes);
                bulk_commit();
            }
            write_row_metadata<kPeer>(p, lane, row, e, wt, d.i, d.w);
            if (slot_lane) bulk_wait_read<1>();  // the previous token's stores have read their stage
            __syncwarp();
            if (lane == 0 && i >= 1) mbar_arrive(&empty[(i - 1) % kBf16Stages]);
        }
        if (slot_lane) bulk_wait_read<0>();  // stages read: the CTA may exit
    }
    __syncthreads();
    if (tid == 0) {
        if (*abort_flag) raise_status(p.status, kDevTimeout);
        finish_tickets(p);
    }
}

int grid_for(const void* kernel, int threads, size_t smem, int64_t work, const DeviceInfo& dev) {
    const int64_t g = static_cast<int64_t>(blocks_per_sm(kernel, dev.device, threads, smem)) *
                      dev.num_sms;
    return static_cast<int>(work < g ? (work > 0 ? work : 1) : g);
}

cudaError_t launch_pdl(const void* kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       const DispatchParams& p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {const_cast<DispatchParams*>(&p)};
    return cudaLaunchKernelExC(&cfg, kernel, args);
}

}  // namespace

cudaError_t launch_dispatch_fp8(const DispatchParams& params, cudaStream_t stream) {
    if (params.T == 0) return cudaSuccess;
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    // Output ring: as many staged rows as fit in 1/kFp8CtasPerSm of the SM's shared
    // memory, so that while the layout kernel runs each SM reads and quantises as
    // many of its tokens as it can hold.
    DispatchParams p = params;
    p.in_stages = kFp8InStages;
    const Fp8Smem one = fp8_smem(p.H, kFp8InStages, 1);
    const Fp8Smem two = fp8_smem(p.H, kFp8InStages, 2);
    const size_t per_out = two.total - one.total;
    size_t budget = dev.smem_per_sm / kFp8CtasPerSm;
    budget = budget > dev.smem_reserved ? budget - dev.smem_reserved : 0;
    if (budget > dev.max_smem_optin) budget = dev.max_smem_optin;
    int no = budget >= one.total ? 1 + static_cast<int>((budget - one.total) / per_out) : 1;
    if (no > kFp8MaxOutStages) no = kFp8MaxOutStages;
    const int ns = fp8_storers(p);
    // a storer releases a stage at its next step: with two storers, ns + 1 stages
    if (no < ns + 1) no = ns + 1;
    p.out_stages = no;
    const Fp8Smem L = fp8_smem(p.H, p.in_stages, p.out_stages);
    if (L.total > dev.max_smem_optin) return cudaErrorInvalidValue;
    const void* kernel =
        p.peer_offset ? (ns == 2 ? reinterpret_cast<const void*>(dispatch_fp8_kernel<true, 2>)
                                 : reinterpret_cast<const void*>(dispatch_fp8_kernel<true, 1>))
                      : (ns == 2 ? reinterpret_cast<const void*>(dispatch_fp8_kernel<false, 2>)
                                 : reinterpret_cast<const void*>(dispatch_fp8_kernel<false, 1>));
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(L.total));
    if (err != cudaSuccess) return err;
    // quantiser warps: at most kFp8MaxQuantWarps, each quantising the same number
    // of block pairs (a row's quantisation is a latency chain per pair, so more
    // warps per row shorten the time a row occupies its stages)
    const int pairs = static_cast<int>((p.H / 128 + 1) / 2);
    const int iters = (pairs + kFp8MaxQuantWarps - 1) / kFp8MaxQuantWarps;
    const int nq = (pairs + iters - 1) / iters;
    const int threads = 32 * (nq + 1 + ns);
    const int grid = grid_for(kernel, threads, L.total, p.T, dev);
    return launch_pdl(kernel, dim3(grid), dim3(threads), L.total, stream, p);
}

cudaError_t launch_dispatch_bf16(const DispatchParams& p, cudaStream_t stream) {
    if (p.T == 0) return cudaSuccess;
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const size_t smem = static_cast<size_t>(kBf16Stages) * p.H * 2 + 16 * kBf16Stages +
                        4 * kTokLog + 16;
    if (smem > dev.max_smem_optin) return cudaErrorInvalidValue;
    const void* kernel = p.peer_offset ? reinterpret_cast<const void*>(dispatch_bf16_kernel<true>)
                                       : reinterpret_cast<const void*>(dispatch_bf16_kernel<false>);
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int grid = grid_for(kernel, 64, smem, p.T, dev);
    return launch_pdl(kernel, dim3(grid), dim3(64), smem, stream, p);
}

}  // namespace ep
