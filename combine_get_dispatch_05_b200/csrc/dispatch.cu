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

constexpr int kFp8Stages = 3;     // input ring depth (tokens in flight per CTA)
constexpr int kFp8OutStages = 2;  // output staging buffers
constexpr int kBf16Stages = 4;

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
    s.off_out = kFp8Stages * s.in_bytes;
    s.off_bars = s.off_out + kFp8OutStages * s.out_bytes;
    s.off_rows = s.off_bars + 8u * kFp8Stages;
    s.off_flag = s.off_rows + 4u * 32u * kFp8OutStages;
    s.total = s.off_flag + 16u;
    return s;
}

__global__ void __launch_bounds__(256) dispatch_fp8_kernel(DispatchParams p) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int64_t T = p.T, H = p.H;
    const int K = p.K, nb = static_cast<int>(H >> 7);
    const Fp8Smem L = fp8_smem(H);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L.off_bars);
    int* rows_sm = reinterpret_cast<int*>(sm + L.off_rows);
    volatile int* abort_flag = reinterpret_cast<int*>(sm + L.off_flag);
    const bool scale_bulk = (static_cast<uint32_t>(nb) * 4u) == L.s_bytes;
    const uint8_t* x = static_cast<const uint8_t*>(p.x);
    uint8_t* recv_x = static_cast<uint8_t*>(p.recv_x);

    const int64_t G = gridDim.x, first = blockIdx.x;
    const int64_t n_mine = first < T ? (T - 1 - first) / G + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < kFp8Stages; ++s) mbar_init(&bars[s], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    int64_t issued = 0;  // loads issued (meaningful in thread 0)
    if (tid == 0) {
        for (; issued < kFp8Stages && issued < n_mine; ++issued) {
            const int64_t t = first + issued * G;
            mbar_arrive_expect_tx(&bars[issued], L.in_bytes);
            bulk_load(sm + issued * L.in_bytes, x + t * H * 2, L.in_bytes, &bars[issued]);
        }
    }

    pdl_wait();  // row_of from the layout kernels is complete and visible

    // warp 0, lane k < K: (row, expert, weight) of slot k, prefetched one token ahead
    int nrow = -1;
    int64_t nexp = -1;
    float nwt = 0.0f;
    const bool slot_lane = (warp == 0) && (lane < K);
    if (slot_lane && n_mine > 0) {
        const int64_t g = first * K + lane;
        nrow = p.row_of[g];
        nexp = p.topk_idx[g];
        nwt = p.topk_weights[g];
    }

    int64_t i = 0;
    for (; i < n_mine; ++i) {
        const int64_t t = first + i * G;
        const int s = static_cast<int>(i % kFp8Stages);
        const uint32_t par = static_cast<uint32_t>((i / kFp8Stages) & 1);
        const int o = static_cast<int>(i % kFp8OutStages);
        uint8_t* out_q = sm + L.off_out + o * L.out_bytes;
        float* out_s = reinterpret_cast<float*>(out_q + L.q_bytes);
        const int row = nrow;
        const int64_t e = nexp;
        const float wt = nwt;
        if (slot_lane) {
            rows_sm[o * 32 + lane] = row;
            if (i + 1 < n_mine) {
                const int64_t g = (t + G) * K + lane;
                nrow = p.row_of[g];
                nexp = p.topk_idx[g];
                nwt = p.topk_weights[g];
            }
            bulk_wait_read<kFp8OutStages - 1>();  // out stage o is no longer being read
        }
        __syncthreads();
        if (!mbar_wait_bounded(&bars[s], par, p.timeout_ns)) *abort_flag = 1;
        quantize_row_fp8(sm + s * L.in_bytes, out_q, out_s, nb, warp, nwarps, lane);
        fence_proxy_async_smem();
        __syncthreads();
        if (*abort_flag) break;
        if (warp == 0) {
            if (lane < K) {
                if (row >= 0) {
                    bulk_store(recv_x + static_cast<int64_t>(row) * H, out_q, L.q_bytes);
                    if (scale_bulk)
                        bulk_store(p.recv_scales + static_cast<int64_t>(row) * nb, out_s,
                                   static_cast<uint32_t>(nb) * 4u);
                    const int64_t epp = p.experts_per_partition;
                    p.recv_topk_idx[row] = static_cast<int32_t>(e - (e / epp) * epp);
                    p.recv_topk_weights[row] = wt;
                }
                bulk_commit();
            }
            __syncwarp();
            // every thread is done reading input stage s: refill it
            if (lane == 0 && issued < n_mine) {
                const int64_t t2 = first + issued * G;
                mbar_arrive_expect_tx(&bars[s], L.in_bytes);
                bulk_load(sm + s * L.in_bytes, x + t2 * H * 2, L.in_bytes, &bars[s]);
                ++issued;
            }
        }
        if (!scale_bulk) {
            for (int idx = tid; idx < K * nb; idx += blockDim.x) {
                const int k = idx / nb, b = idx - k * nb;
                const int r = rows_sm[o * 32 + k];
                if (r >= 0) p.recv_scales[static_cast<int64_t>(r) * nb + b] = out_s[b];
            }
        }
    }
    if (i < n_mine && tid == 0) {
        // a bounded wait gave up: report, then let the loads still in flight land
        // before this CTA's shared memory goes away
        raise_status(p.status, kDevTimeout);
        for (int64_t j = i; j < issued; ++j)
            mbar_wait_bounded(&bars[j % kFp8Stages],
                              static_cast<uint32_t>((j / kFp8Stages) & 1), kDefaultTimeoutNs);
    }
    if (slot_lane) bulk_wait_all<0>();
}

__global__ void __launch_bounds__(32) dispatch_bf16_kernel(DispatchParams p) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int lane = threadIdx.x;
    const int64_t T = p.T, H = p.H;
    const int K = p.K;
    const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kBf16Stages * row_bytes);
    const uint8_t* x = static_cast<const uint8_t*>(p.x);
    uint8_t* recv_x = static_cast<uint8_t*>(p.recv_x);

    const int64_t G = gridDim.x, first = blockIdx.x;
    const int64_t n_mine = first < T ? (T - 1 - first) / G + 1 : 0;

    if (lane == 0) {
        for (int s = 0; s < kBf16Stages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    int64_t issued = 0;
    if (lane == 0) {
        for (; issued < kBf16Stages && issued < n_mine; ++issued) {
            const int64_t t = first + issued * G;
            mbar_arrive_expect_tx(&bars[issued], row_bytes);
            bulk_load(sm + issued * row_bytes, x + t * row_bytes, row_bytes, &bars[issued]);
        }
    }

    pdl_wait();

    const bool slot_lane = lane < K;
    int nrow = -1;
    int64_t nexp = -1;
    float nwt = 0.0f;
    if (slot_lane && n_mine > 0) {
        const int64_t g = first * K + lane;
        nrow = p.row_of[g];
        nexp = p.topk_idx[g];
        nwt = p.topk_weights[g];
    }

    int64_t i = 0;
    bool aborted = false;
    for (; i < n_mine; ++i) {
        const int64_t t = first + i * G;
        const int s = static_cast<int>(i % kBf16Stages);
        const uint32_t par = static_cast<uint32_t>((i / kBf16Stages) & 1);
        const int row = nrow;
        const int64_t e = nexp;
        const float wt = nwt;
        if (slot_lane && i + 1 < n_mine) {
            const int64_t g = (t + G) * K + lane;
            nrow = p.row_of[g];
            nexp = p.topk_idx[g];
            nwt = p.topk_weights[g];
        }
        const bool ok = mbar_wait_bounded(&bars[s], par, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) {
            aborted = true;
            break;
        }
        if (slot_lane) {
            if (row >= 0) {
                bulk_store(recv_x + static_cast<int64_t>(row) * row_bytes, sm + s * row_bytes,
                           row_bytes);
                const int64_t epp = p.experts_per_partition;
                p.recv_topk_idx[row] = static_cast<int32_t>(e - (e / epp) * epp);
                p.recv_topk_weights[row] = wt;
            }
            bulk_commit();
            bulk_wait_read<1>();  // this lane's stores of token i-1 have read their stage
        }
        __syncwarp();
        // stage of token i-1 is free: refill it with the next token of this CTA
        if (lane == 0 && i >= 1 && issued < n_mine) {
            const int ps = static_cast<int>((i - 1) % kBf16Stages);
            const int64_t t2 = first + issued * G;
            mbar_arrive_expect_tx(&bars[ps], row_bytes);
            bulk_load(sm + ps * row_bytes, x + t2 * row_bytes, row_bytes, &bars[ps]);
            ++issued;
        }
    }
    if (aborted && lane == 0) {
        raise_status(p.status, kDevTimeout);
        for (int64_t j = i; j < issued; ++j)
            mbar_wait_bounded(&bars[j % kBf16Stages], static_cast<uint32_t>((j / kBf16Stages) & 1),
                              kDefaultTimeoutNs);
    }
    if (slot_lane) bulk_wait_all<0>();
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
    // warps: enough that every warp quantises the same number of block pairs
    const int pairs = static_cast<int>((p.H / 128 + 1) / 2);
    const int iters = (pairs + 7) / 8;
    const int warps = (pairs + iters - 1) / iters;
    const int threads = 32 * (warps > 0 ? warps : 1);
    const int grid = grid_for(kernel, threads, L.total, p.T, dev.num_sms);
    return launch_pdl(kernel, dim3(grid), dim3(threads), L.total, stream, p);
}

cudaError_t launch_dispatch_bf16(const DispatchParams& p, cudaStream_t stream) {
    if (p.T == 0) return cudaSuccess;
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const size_t smem = static_cast<size_t>(kBf16Stages) * p.H * 2 + 8 * kBf16Stages;
    if (smem > dev.max_smem_optin) return cudaErrorInvalidValue;
    const void* kernel = reinterpret_cast<const void*>(dispatch_bf16_kernel);
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int grid = grid_for(kernel, 32, smem, p.T, dev.num_sms);
    return launch_pdl(kernel, dim3(grid), dim3(32), smem, stream, p);
}

}  // namespace ep
