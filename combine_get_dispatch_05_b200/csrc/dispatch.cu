// dispatch.cu -- write every token to each of its receive rows.
//
// FP8 path ("DeepSeek 开源周第二弹：DeepEP", sections "DeepEP 的核心功能" (native FP8)
// and "DeepEP 的常规内核和低延迟内核" (FP8 dispatch)): per token, per 128-channel
// block, amax -> scale s = max(amax, 1e-4) / 448 -> q = e4m3_rne_satfinite(x / s);
// the E4M3 row and its fp32 scales go to every row_of[t, k].
//
// BF16 path: the row is copied bit for bit.
//
// Both kernels are persistent pipelines over the CTA's tokens (t = blockIdx.x,
// blockIdx.x + gridDim.x, ...).  Input rows arrive by 1-D bulk async copies
// (cp.async.bulk, mbarrier completion) into a ring of shared-memory stages, so
// several 14 KB rows per SM are in flight from HBM at once; output rows leave by
// bulk stores from shared memory, one per destination row, issued by one lane
// per top-k slot.  A token is read from HBM once and written K times: the
// traffic is the algorithmic minimum.  The x loads of the first stages are
// issued before waiting on the layout kernels (x is an input of the call), so
// they overlap the layout.
#include "ep_device.cuh"
#include "ep_internal.h"
#include "ep_quant.cuh"

namespace ep {

namespace {

constexpr int kFp8InStages = 3;   // input ring: rows in flight from HBM per CTA
constexpr int kFp8OutStages = 3;  // quantised rows staged for the bulk stores
constexpr int kBf16Stages = 4;    // BF16 rows in flight per CTA

struct Fp8Smem {
    uint32_t in_bytes, q_bytes, s_bytes, out_bytes;
    uint32_t off_out, off_bars, off_rows, off_flag, total;
};

__host__ __device__ inline Fp8Smem fp8_smem(int64_t H) {
    Fp8Smem s;
    const uint32_t nb = static_cast<uint32_t>(H / 128);
    s.in_bytes = static_cast<uint32_t>(H) * 2u;
    s.q_bytes = static_cast<uint32_t>(H);
    s.s_bytes = (nb * 4u + 15u) & ~15u;
    s.out_bytes = s.q_bytes + s.s_bytes;
    s.off_out = kFp8InStages * s.in_bytes;
    s.off_bars = s.off_out + kFp8OutStages * s.out_bytes;
    s.off_rows = s.off_bars + 8u * 2u * (kFp8InStages + kFp8OutStages);
    s.off_flag = s.off_rows + 4u * 32u * kFp8OutStages;
    s.total = s.off_flag + 16u;
    return s;
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

// Metadata of one token's receive rows, written by the storer warp.  Per-expert
// rows: lane k owns slot k and writes the local id and weight of its row.
// Deduplicated rows (one per partition): lane p owns partition p's row and writes
// its K-entry lists, reading every slot's id and weight from the id lanes by
// shuffle (all lanes take part in the shuffles).
__device__ __forceinline__ void write_row_metadata(const DispatchParams& p, int lane, int row,
                                                   int64_t e, float wt) {
    const int64_t epp = p.experts_per_partition;
    if (!p.dedup) {
        if (lane < p.slots && row >= 0) {
            p.recv_topk_idx[row] = static_cast<int32_t>(e - (e / epp) * epp);
            p.recv_topk_weights[row] = wt;
        }
        return;
    }
    for (int k = 0; k < p.K; ++k) {
        const int64_t ek = __shfl_sync(0xffffffffu, e, k);
        const float wk = __shfl_sync(0xffffffffu, wt, k);
        if (lane < p.slots && row >= 0) {
            const bool in = ek >= 0 && ek < p.num_experts && ek / epp == lane;
            p.recv_topk_idx[static_cast<int64_t>(row) * p.K + k] =
                in ? static_cast<int32_t>(ek - lane * epp) : -1;
            p.recv_topk_weights[static_cast<int64_t>(row) * p.K + k] = in ? wk : 0.0f;
        }
    }
}

// Warp-specialised pipeline, one CTA = 1 loader warp + nq quantiser warps + 1 storer
// warp, coupled only by mbarriers (no CTA-wide barrier after set-up):
//   loader (warp 0, lane 0): bulk-loads token rows into the input ring
//       (in_full[s]: transaction bytes; waits in_empty[s] before reusing a stage);
//   quantisers (warps 1..nq): quantise their share of the row's 128-channel blocks
//       from input stage s into output stage o, then arrive on in_empty[s] and
//       out_full[o] (waiting out_empty[o] before reusing an output stage);
//   storer (last warp): lane k bulk-stores the staged row and its scales to row
//       row_of[t, k], writes recv_topk_idx / recv_topk_weights, and releases the
//       output stage (out_empty) once its stores have read it.
// Only the storer reads what the layout kernel wrote, so only it waits on the
// programmatic dependency; loads and quantisation overlap the layout.
__global__ void __launch_bounds__(352) dispatch_fp8_kernel(DispatchParams p) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nq = (blockDim.x >> 5) - 2;
    const int64_t T = p.T, H = p.H;
    const int K = p.K, nb = static_cast<int>(H >> 7);
    const Fp8Smem L = fp8_smem(H);
    uint64_t* in_full = reinterpret_cast<uint64_t*>(sm + L.off_bars);
    uint64_t* in_empty = in_full + kFp8InStages;
    uint64_t* out_full = in_empty + kFp8InStages;
    uint64_t* out_empty = out_full + kFp8OutStages;
    int* rows_sm = reinterpret_cast<int*>(sm + L.off_rows);
    volatile int* abort_flag = reinterpret_cast<int*>(sm + L.off_flag);
    const bool scale_bulk = (static_cast<uint32_t>(nb) * 4u) == L.s_bytes;

    const int64_t G = gridDim.x, first = blockIdx.x;
    const int64_t n_mine = first < T ? (T - 1 - first) / G + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < kFp8InStages; ++s) {
            mbar_init(&in_full[s], 1);
            mbar_init(&in_empty[s], nq);
        }
        for (int o = 0; o < kFp8OutStages; ++o) {
            mbar_init(&out_full[o], nq);
            mbar_init(&out_empty[o], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- loader
        if (lane == 0) {
            const uint8_t* x = static_cast<const uint8_t*>(p.x);
            int64_t issued = 0;
            for (; issued < n_mine; ++issued) {
                const int s = static_cast<int>(issued % kFp8InStages);
                if (issued >= kFp8InStages &&
                    !wait_or_abort(&in_empty[s],
                                   static_cast<uint32_t>((issued / kFp8InStages - 1) & 1),
                                   p.timeout_ns, abort_flag))
                    break;
                const int64_t t = first + issued * G;
                mbar_arrive_expect_tx(&in_full[s], L.in_bytes);
                bulk_load(sm + s * L.in_bytes, x + t * H * 2, L.in_bytes, &in_full[s]);
            }
            if (*abort_flag) {
                // let this CTA's loads still in flight land before it exits: the
                // latest load of each stage is its barrier's current phase
                for (int64_t j = issued - 1; j >= 0 && j >= issued - kFp8InStages; --j)
                    mbar_wait_bounded(&in_full[j % kFp8InStages],
                                      static_cast<uint32_t>((j / kFp8InStages) & 1),
                                      kDefaultTimeoutNs);
            }
        }
    } else if (warp <= nq) {
        // ------------------------------------------------------------ quantisers
        const int qw = warp - 1;
        for (int64_t i = 0; i < n_mine; ++i) {
            const int s = static_cast<int>(i % kFp8InStages);
            const int o = static_cast<int>(i % kFp8OutStages);
            if (!wait_or_abort(&in_full[s], static_cast<uint32_t>((i / kFp8InStages) & 1),
                               p.timeout_ns, abort_flag))
                break;
            if (i >= kFp8OutStages &&
                !wait_or_abort(&out_empty[o], static_cast<uint32_t>((i / kFp8OutStages - 1) & 1),
                               p.timeout_ns, abort_flag))
                break;
            uint8_t* out_q = sm + L.off_out + o * L.out_bytes;
            quantize_row_fp8(sm + s * L.in_bytes, out_q, reinterpret_cast<float*>(out_q + L.q_bytes),
                             nb, qw, nq, lane, p.pow2_scales != 0);
            fence_proxy_async_smem();  // staged row visible to the bulk stores
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&in_empty[s]);
                mbar_arrive(&out_full[o]);
            }
        }
    } else {
        // ---------------------------------------------------------------- storer
        pdl_wait();  // row_of from the layout kernel is complete and visible
        uint8_t* recv_x = static_cast<uint8_t*>(p.recv_x);
        const int S = p.slots;
        const bool slot_lane = lane < S;  // lane s stores slot s's row
        const bool id_lane = lane < K;    // lane k holds routing entry k
        int nrow = -1;
        int64_t nexp = -1;
        float nwt = 0.0f;
        if (n_mine > 0) {
            if (slot_lane) nrow = p.row_of[first * S + lane];
            if (id_lane) {
                nexp = p.topk_idx[first * K + lane];
                nwt = p.topk_weights[first * K + lane];
            }
        }
        for (int64_t i = 0; i < n_mine; ++i) {
            const int64_t t = first + i * G;
            const int o = static_cast<int>(i % kFp8OutStages);
            const int row = nrow;
            const int64_t e = nexp;
            const float wt = nwt;
            if (i + 1 < n_mine) {
                if (slot_lane) nrow = p.row_of[(t + G) * S + lane];
                if (id_lane) {
                    nexp = p.topk_idx[(t + G) * K + lane];
                    nwt = p.topk_weights[(t + G) * K + lane];
                }
            }
            if (!wait_or_abort(&out_full[o], static_cast<uint32_t>((i / kFp8OutStages) & 1),
                               p.timeout_ns, abort_flag))
                break;
            uint8_t* out_q = sm + L.off_out + o * L.out_bytes;
            const float* out_s = reinterpret_cast<const float*>(out_q + L.q_bytes);
            if (slot_lane) {
                if (row >= 0) {
                    bulk_store(recv_x + static_cast<int64_t>(row) * H, out_q, L.q_bytes);
                    if (scale_bulk)
                        bulk_store(p.recv_scales + static_cast<int64_t>(row) * nb, out_s,
                                   static_cast<uint32_t>(nb) * 4u);
                }
                bulk_commit();
                rows_sm[o * 32 + lane] = row;
            }
            write_row_metadata(p, lane, row, e, wt);
            if (!scale_bulk) {
                __syncwarp();
                for (int idx = lane; idx < S * nb; idx += 32) {
                    const int k = idx / nb, b = idx - k * nb;
                    const int r = rows_sm[o * 32 + k];
                    if (r >= 0) p.recv_scales[static_cast<int64_t>(r) * nb + b] = out_s[b];
                }
            }
            // release the previous output stage once this warp's stores have read it
            if (slot_lane) bulk_wait_read<1>();
            __syncwarp();
            if (lane == 0 && i >= 1) mbar_arrive(&out_empty[(i - 1) % kFp8OutStages]);
        }
        if (slot_lane) bulk_wait_all<0>();
    }
    if (tid == 0 && *abort_flag) raise_status(p.status, kDevTimeout);
}

// BF16 rows are copied bit for bit, so the row staged by the bulk load is itself
// the source of the K bulk stores.  One CTA = a loader warp and a storer warp
// coupled by full/empty mbarriers over a ring of kBf16Stages rows:
//   loader (warp 0, lane 0): waits empty[s], bulk-loads the next token's row into
//       stage s (full[s] counts its transaction bytes);
//   storer (warp 1): waits for the layout, then per token waits full[s], lane k
//       bulk-stores the row to row_of[t, k] and writes recv_topk_idx / weights;
//       once this token's stores have read the stage it arrives on empty[s].
__global__ void __launch_bounds__(64) dispatch_bf16_kernel(DispatchParams p) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t T = p.T, H = p.H;
    const int K = p.K;
    const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kBf16Stages * row_bytes);
    uint64_t* empty = full + kBf16Stages;
    volatile int* abort_flag = reinterpret_cast<int*>(empty + kBf16Stages);

    const int64_t G = gridDim.x, first = blockIdx.x;
    const int64_t n_mine = first < T ? (T - 1 - first) / G + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < kBf16Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- loader
        if (lane == 0) {
            const uint8_t* x = static_cast<const uint8_t*>(p.x);
            int64_t issued = 0;
            for (; issued < n_mine; ++issued) {
                const int s = static_cast<int>(issued % kBf16Stages);
                if (issued >= kBf16Stages &&
                    !wait_or_abort(&empty[s], static_cast<uint32_t>((issued / kBf16Stages - 1) & 1),
                                   p.timeout_ns, abort_flag))
                    break;
                const int64_t t = first + issued * G;
                mbar_arrive_expect_tx(&full[s], row_bytes);
                bulk_load(sm + s * row_bytes, x + t * row_bytes, row_bytes, &full[s]);
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
        const bool id_lane = lane < K;    // lane k holds routing entry k
        int nrow = -1;
        int64_t nexp = -1;
        float nwt = 0.0f;
        if (n_mine > 0) {
            if (slot_lane) nrow = p.row_of[first * S + lane];
            if (id_lane) {
                nexp = p.topk_idx[first * K + lane];
                nwt = p.topk_weights[first * K + lane];
            }
        }
        for (int64_t i = 0; i < n_mine; ++i) {
            const int64_t t = first + i * G;
            const int s = static_cast<int>(i % kBf16Stages);
            const int row = nrow;
            const int64_t e = nexp;
            const float wt = nwt;
            if (i + 1 < n_mine) {
                if (slot_lane) nrow = p.row_of[(t + G) * S + lane];
                if (id_lane) {
                    nexp = p.topk_idx[(t + G) * K + lane];
                    nwt = p.topk_weights[(t + G) * K + lane];
                }
            }
            if (!wait_or_abort(&full[s], static_cast<uint32_t>((i / kBf16Stages) & 1), p.timeout_ns,
                               abort_flag))
                break;
            if (slot_lane) {
                if (row >= 0)
                    bulk_store(recv_x + static_cast<int64_t>(row) * row_bytes, sm + s * row_bytes,
                               row_bytes);
                bulk_commit();
            }
            write_row_metadata(p, lane, row, e, wt);
            if (slot_lane) bulk_wait_read<1>();  // the previous token's stores have read their stage
            __syncwarp();
            if (lane == 0 && i >= 1) mbar_arrive(&empty[(i - 1) % kBf16Stages]);
        }
        if (slot_lane) bulk_wait_all<0>();
    }
    if (tid == 0 && *abort_flag) raise_status(p.status, kDevTimeout);
}

int grid_for(const void* kernel, int threads, size_t smem, int64_t work, int num_sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t g = static_cast<int64_t>(per_sm) * num_sms;
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

cudaError_t launch_dispatch_fp8(const DispatchParams& p, cudaStream_t stream) {
    if (p.T == 0) return cudaSuccess;
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const Fp8Smem L = fp8_smem(p.H);
    if (L.total > dev.max_smem_optin) return cudaErrorInvalidValue;
    const void* kernel = reinterpret_cast<const void*>(dispatch_fp8_kernel);
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(L.total));
    if (err != cudaSuccess) return err;
    // quantiser warps: enough that each quantises the same number of block pairs
    const int pairs = static_cast<int>((p.H / 128 + 1) / 2);
    const int iters = (pairs + 7) / 8;
    const int nq = (pairs + iters - 1) / iters;
    const int threads = 32 * (nq + 2);
    const int grid = grid_for(kernel, threads, L.total, p.T, dev.num_sms);
    return launch_pdl(kernel, dim3(grid), dim3(threads), L.total, stream, p);
}

cudaError_t launch_dispatch_bf16(const DispatchParams& p, cudaStream_t stream) {
    if (p.T == 0) return cudaSuccess;
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const size_t smem = static_cast<size_t>(kBf16Stages) * p.H * 2 + 16 * kBf16Stages + 16;
    if (smem > dev.max_smem_optin) return cudaErrorInvalidValue;
    const void* kernel = reinterpret_cast<const void*>(dispatch_bf16_kernel);
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int grid = grid_for(kernel, 64, smem, p.T, dev.num_sms);
    return launch_pdl(kernel, dim3(grid), dim3(64), smem, stream, p);
}

}  // namespace ep
