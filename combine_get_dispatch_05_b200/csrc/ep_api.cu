// ep_api.cu -- the exported C ABI (include/ep_b200.h): host-side argument checks,
// workspace handling and kernel launches.  No allocation (except ep_ipc_alloc), no
// host synchronisation except in ep_read_status().
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "ep_b200.h"
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_have_info[kMaxDevices];
DeviceInfo g_info[kMaxDevices];

struct OccupancyEntry {
    const void* kernel;
    int device, threads;
    size_t smem;
    int per_sm;
};
constexpr int kOccupancyEntries = 64;
std::mutex g_occ_mu;
OccupancyEntry g_occ[kOccupancyEntries];
int g_occ_n = 0;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ep_status check_hidden(int64_t H, bool fp8) {
    if (H <= 0 || H > 16384) return EP_ERR_SHAPE;
    if (fp8 ? (H % 128 != 0) : (H % 8 != 0)) return EP_ERR_SHAPE;
    return EP_OK;
}

inline ep_status cuda_status(cudaError_t e) { return e == cudaSuccess ? EP_OK : EP_ERR_CUDA; }

}  // namespace

// Argument checks shared by every layout entry point (ep_internal.h).
ep_status check_routing(int64_t T, int32_t K, int32_t E, int32_t P) {
    if (T < 0 || K < 1 || K > 32 || E < 1 || E > 4096 || P < 1 || P > 64 || E % P != 0)
        return EP_ERR_SHAPE;
    if (T * static_cast<int64_t>(K) >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    return EP_OK;
}

ep_status check_layout_ptrs(const ep_layout* lay, int64_t T) {
    if (!lay || !lay->num_tokens_per_expert || !lay->num_tokens_per_partition ||
        !lay->expert_offset || !lay->num_recv)
        return EP_ERR_INVALID_ARG;
    if (T > 0 && (!lay->is_token_in_partition || !lay->row_of || !lay->src_of))
        return EP_ERR_INVALID_ARG;
    return EP_OK;
}

// EP_ERR_SHAPE if the batch is too large for the layout kernels.
ep_status check_layout_size(int64_t T, int32_t K, int32_t E, int32_t P, bool by_partition) {
    bool fits = true;
    if (layout_fits(T, K, E, P, by_partition, &fits) != cudaSuccess) return EP_ERR_CUDA;
    return fits ? EP_OK : EP_ERR_SHAPE;
}

int blocks_per_sm(const void* kernel, int device, int threads, size_t smem) {
    std::lock_guard<std::mutex> lock(g_occ_mu);
    for (int i = 0; i < g_occ_n; ++i) {
        const OccupancyEntry& o = g_occ[i];
        if (o.kernel == kernel && o.device == device && o.threads == threads && o.smem == smem)
            return o.per_sm;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) !=
        cudaSuccess)
        return 1;  // not kept: the launch that follows reports the error
    if (per_sm < 1) per_sm = 1;
    if (g_occ_n < kOccupancyEntries) g_occ[g_occ_n++] = {kernel, device, threads, smem, per_sm};
    return per_sm;
}

cudaError_t device_info(DeviceInfo* out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < kMaxDevices && g_have_info[dev].load(std::memory_order_acquire)) {
        *out = g_info[dev];
        return cudaSuccess;
    }
    DeviceInfo d;
    d.device = dev;
    err = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    int optin = 0;
    err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err != cudaSuccess) return err;
    d.max_smem_optin = static_cast<size_t>(optin);
    int per_sm = 0, reserved = 0;
    err = cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (err != cudaSuccess) return err;
    d.smem_per_sm = static_cast<size_t>(per_sm);
    d.smem_reserved = static_cast<size_t>(reserved);
    if (dev >= 0 && dev < kMaxDevices) {
        g_info[dev] = d;
        g_have_info[dev].store(1, std::memory_order_release);
    }
    *out = d;
    return cudaSuccess;
}

}  // namespace ep

using namespace ep;

extern "C" {

int32_t ep_abi_version(void) { return 2; }

const char* ep_status_string(int32_t status) {
    switch (status) {
        case EP_OK: return "ok";
        case EP_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, unknown enum)";
        case EP_ERR_SHAPE: return "unsupported size";
        case EP_ERR_WORKSPACE: return "workspace too small";
        case EP_ERR_CUDA: return "CUDA runtime error";
        default: return "unknown status";
    }
}

size_t ep_workspace_bytes(int64_t num_tokens, int32_t num_experts, int32_t num_partitions) {
    if (num_tokens < 0 || num_experts < 1 || num_partitions < 1) return 0;
    const size_t body = sizeof(int32_t) * static_cast<size_t>(max_layout_chunks(num_tokens)) *
                        (static_cast<size_t>(num_experts) + static_cast<size_t>(num_partitions));
    return (kWsHeader + body + 255) / 256 * 256;
}

ep_status ep_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace || workspace_bytes < kWsHeader) return EP_ERR_INVALID_ARG;
    return cuda_status(
        cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)));
}

ep_status ep_read_status(void* workspace, size_t workspace_bytes, void* stream, uint32_t* bits_out) {
    if (!workspace || !bits_out || workspace_bytes < kWsHeader) return EP_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t bits = 0;
    cudaError_t err = cudaMemcpyAsync(&bits, static_cast<uint8_t*>(workspace) + kWsStatus,
                                      sizeof(bits), cudaMemcpyDeviceToHost, s);
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    if (err == cudaSuccess)
        err = cudaMemsetAsync(static_cast<uint8_t*>(workspace) + kWsStatus, 0, sizeof(uint32_t), s);
    if (err != cudaSuccess) return EP_ERR_CUDA;
    *bits_out = bits;
    return EP_OK;
}

ep_status ep_get_dispatch_layout(int64_t num_tokens, int32_t num_topk, int32_t num_experts,
                                 int32_t num_partitions, const int64_t* topk_idx,
                                 const ep_layout* layout, void* workspace, size_t workspace_bytes,
                                 void* stream) {
    ep_status st = check_routing(num_tokens, num_topk, num_experts, num_partitions);
    if (st != EP_OK) return st;
    if ((st = check_layout_ptrs(layout, num_tokens)) != EP_OK) return st;
    if (!workspace || !aligned16(workspace) || (num_tokens > 0 && !topk_idx))
        return EP_ERR_INVALID_ARG;
    if (workspace_bytes < ep_workspace_bytes(num_tokens, num_experts, num_partitions))
        return EP_ERR_WORKSPACE;
    if ((st = check_layout_size(num_tokens, num_topk, num_experts, num_partitions, false)) != EP_OK)
        return st;
    const Workspace ws = carve_workspace(workspace, num_tokens, num_experts);
    return cuda_status(launch_layout(num_tokens, num_topk, num_experts, num_partitions, topk_idx,
                                     *layout, ws, static_cast<cudaStream_t>(stream)));
}

ep_status ep_dispatch(int64_t num_tokens, int64_t hidden, int32_t num_topk, int32_t num_experts,
                      int32_t num_partitions, int32_t quant, const void* x, const int64_t* topk_idx,
                      const float* topk_weights, void* recv_x, float* recv_scales,
                      int32_t* recv_topk_idx, float* recv_topk_weights, const ep_layout* handle,
                      void* workspace, size_t workspace_bytes, void* stream) {
    const bool scales_mn = (quant & EP_QUANT_SCALES_MN_MAJOR) != 0;
    quant &= ~EP_QUANT_SCALES_MN_MAJOR;
    if (quant != EP_QUANT_NONE && quant != EP_QUANT_FP8_E4M3_1X128 &&
        quant != EP_QUANT_FP8_E4M3_1X128_POW2)
        return EP_ERR_INVALID_ARG;
    const bool fp8 = quant != EP_QUANT_NONE;
    if (scales_mn && !fp8) return EP_ERR_INVALID_ARG;  // BF16 rows carry no scales
    ep_status st = check_routing(num_tokens, num_topk, num_experts, num_partitions);
    if (st != EP_OK) return st;
    if ((st = check_hidden(hidden, fp8)) != EP_OK) return st;
    if ((st = check_layout_ptrs(handle, num_tokens)) != EP_OK) return st;
    if (!workspace || !aligned16(workspace)) return EP_ERR_INVALID_ARG;
    if (num_tokens > 0) {
        if (!x || !topk_idx || !topk_weights || !recv_x || !recv_topk_idx || !recv_topk_weights)
            return EP_ERR_INVALID_ARG;
        if (fp8 && !recv_scales) return EP_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(recv_x) || (fp8 && !aligned16(recv_scales)))
            return EP_ERR_INVALID_ARG;
    }
    if (workspace_bytes < ep_workspace_bytes(num_tokens, num_experts, num_partitions))
        return EP_ERR_WORKSPACE;
    if ((st = check_layout_size(num_tokens, num_topk, num_experts, num_partitions, false)) != EP_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Workspace ws = carve_workspace(workspace, num_tokens, num_experts);
    cudaError_t err =
        launch_layout(num_tokens, num_topk, num_experts, num_partitions, topk_idx, *handle, ws, s);
    if (err != cudaSuccess) return EP_ERR_CUDA;
    DispatchParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.slots = num_topk;
    p.dedup = 0;
    p.pow2_scales = quant == EP_QUANT_FP8_E4M3_1X128_POW2 ? 1 : 0;
    p.scales_mn = scales_mn ? 1 : 0;
    p.scales_ld = (num_tokens * num_topk + 3) / 4 * 4;
    p.num_experts = num_experts;
    p.experts_per_partition = num_experts / num_partitions;
    p.x = x;
    p.topk_idx = topk_idx;
    p.topk_weights = topk_weights;
    p.row_of = handle->row_of;
    p.recv_x = recv_x;
    p.recv_scales = recv_scales;
    p.recv_topk_idx = recv_topk_idx;
    p.recv_topk_weights = recv_topk_weights;
    p.status = ws.status;
    p.ticket = ws.ticket;
    p.done = ws.done;
    p.timeout_ns = kDefaultTimeoutNs;
    return cuda_status(fp8 ? launch_dispatch_fp8(p, s) : launch_dispatch_bf16(p, s));
}

ep_status ep_combine(int64_t num_tokens, int64_t hidden, int32_t num_topk, const void* expert_out,
                     int64_t expert_out_rows, const ep_layout* handle, const float* topk_weights,
                     void* y, void* workspace, size_t workspace_bytes, void* stream) {
    if (num_tokens < 0 || num_topk < 1 || num_topk > 32 || expert_out_rows < 0) return EP_ERR_SHAPE;
    if (num_tokens * static_cast<int64_t>(num_topk) >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    ep_status st = check_hidden(hidden, false);
    if (st != EP_OK) return st;
    if (!handle || !workspace || workspace_bytes < kWsHeader) return EP_ERR_INVALID_ARG;
    if (num_tokens == 0) return EP_OK;
    if (!handle->row_of || !topk_weights || !y || (!expert_out && expert_out_rows > 0))
        return EP_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(expert_out)) return EP_ERR_INVALID_ARG;
    CombineParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.expert_out = expert_out;
    p.expert_out_rows = expert_out_rows;
    p.row_of = handle->row_of;
    p.topk_weights = topk_weights;
    p.y = y;
    p.grad_recv_w = nullptr;
    p.grad_w = nullptr;
    p.status = carve_workspace(workspace, 0, 1).status;
    return cuda_status(launch_combine(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_dispatch_dedup(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                            int32_t num_experts, int32_t num_partitions, int32_t quant,
                            const void* x, const int64_t* topk_idx, const float* topk_weights,
                            void* recv_x, float* recv_scales, int32_t* recv_topk_idx,
                            float* recv_topk_weights, const ep_layout* handle, void* workspace,
                            size_t workspace_bytes, void* stream) {
    const bool scales_mn = (quant & EP_QUANT_SCALES_MN_MAJOR) != 0;
    quant &= ~EP_QUANT_SCALES_MN_MAJOR;
    if (quant != EP_QUANT_NONE && quant != EP_QUANT_FP8_E4M3_1X128 &&
        quant != EP_QUANT_FP8_E4M3_1X128_POW2)
        return EP_ERR_INVALID_ARG;
    const bool fp8 = quant != EP_QUANT_NONE;
    if (scales_mn && !fp8) return EP_ERR_INVALID_ARG;  // BF16 rows carry no scales
    ep_status st = check_routing(num_tokens, num_topk, num_experts, num_partitions);
    if (st != EP_OK) return st;
    if (num_partitions > 32) return EP_ERR_SHAPE;  // one storer lane per partition
    if (num_tokens * static_cast<int64_t>(num_partitions) >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    if ((st = check_hidden(hidden, fp8)) != EP_OK) return st;
    if ((st = check_layout_ptrs(handle, num_tokens)) != EP_OK) return st;
    if (!workspace || !aligned16(workspace)) return EP_ERR_INVALID_ARG;
    if (num_tokens > 0) {
        if (!x || !topk_idx || !topk_weights || !recv_x || !recv_topk_idx || !recv_topk_weights)
            return EP_ERR_INVALID_ARG;
        if (fp8 && !recv_scales) return EP_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(recv_x) || (fp8 && !aligned16(recv_scales)))
            return EP_ERR_INVALID_ARG;
    }
    if (workspace_bytes < ep_workspace_bytes(num_tokens, num_experts, num_partitions))
        return EP_ERR_WORKSPACE;
    if ((st = check_layout_size(num_tokens, num_topk, num_experts, num_partitions, true)) != EP_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Workspace ws = carve_workspace(workspace, num_tokens, num_partitions);
    cudaError_t err = launch_layout(num_tokens, num_topk, num_experts, num_partitions, topk_idx,
                                    *handle, ws, s, /*by_partition=*/true);
    if (err != cudaSuccess) return EP_ERR_CUDA;
    DispatchParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.slots = num_partitions;
    p.dedup = 1;
    p.pow2_scales = quant == EP_QUANT_FP8_E4M3_1X128_POW2 ? 1 : 0;
    p.scales_mn = scales_mn ? 1 : 0;
    p.scales_ld = (num_tokens * (num_partitions < num_topk ? num_partitions : num_topk) + 3) / 4 * 4;
    p.num_experts = num_experts;
    p.experts_per_partition = num_experts / num_partitions;
    p.x = x;
    p.topk_idx = topk_idx;
    p.topk_weights = topk_weights;
    p.row_of = handle->row_of;
    p.recv_x = recv_x;
    p.recv_scales = recv_scales;
    p.recv_topk_idx = recv_topk_idx;
    p.recv_topk_weights = recv_topk_weights;
    p.status = ws.status;
    p.ticket = ws.ticket;
    p.done = ws.done;
    p.timeout_ns = kDefaultTimeoutNs;
    return cuda_status(fp8 ? launch_dispatch_fp8(p, s) : launch_dispatch_bf16(p, s));
}

ep_status ep_combine_dedup(int64_t num_tokens, int64_t hidden, int32_t num_partitions,
                           const void* partition_out, int64_t partition_out_rows,
                           const ep_layout* handle, void* y, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (num_tokens < 0 || num_partitions < 1 || num_partitions > 32 || partition_out_rows < 0)
        return EP_ERR_SHAPE;
    if (num_tokens * static_cast<int64_t>(num_partitions) >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    ep_status st = check_hidden(hidden, false);
    if (st != EP_OK) return st;
    if (!handle || !workspace || !aligned16(workspace) || workspace_bytes < kWsHeader)
        return EP_ERR_INVALID_ARG;
    if (num_tokens == 0) return EP_OK;
    if (!handle->row_of || !y || (!partition_out && partition_out_rows > 0))
        return EP_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(partition_out)) return EP_ERR_INVALID_ARG;
    CombineParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_partitions;  // slots are partitions
    p.expert_out = partition_out;
    p.expert_out_rows = partition_out_rows;
    p.row_of = handle->row_of;
    p.topk_weights = nullptr;  // partitions return weighted rows: a plain sum
    p.y = y;
    p.grad_recv_w = nullptr;
    p.grad_w = nullptr;
    p.status = carve_workspace(workspace, 0, 1).status;
    p.sparse = 1;  // a token reaches few of the P partitions
    return cuda_status(launch_combine(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_dispatch_backward(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                               const void* grad_recv_x, int64_t grad_recv_rows,
                               const ep_layout* handle, const float* grad_recv_topk_weights,
                               void* grad_x, float* grad_topk_weights, void* workspace,
                               size_t workspace_bytes, void* stream) {
    if (num_tokens < 0 || num_topk < 1 || num_topk > 32 || grad_recv_rows < 0) return EP_ERR_SHAPE;
    if (num_tokens * static_cast<int64_t>(num_topk) >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    ep_status st = check_hidden(hidden, false);
    if (st != EP_OK) return st;
    if (!handle || !workspace || !aligned16(workspace) || workspace_bytes < kWsHeader)
        return EP_ERR_INVALID_ARG;
    if ((grad_recv_topk_weights == nullptr) != (grad_topk_weights == nullptr))
        return EP_ERR_INVALID_ARG;
    if (num_tokens == 0) return EP_OK;
    if (!handle->row_of || !grad_x || (!grad_recv_x && grad_recv_rows > 0)) return EP_ERR_INVALID_ARG;
    if (!aligned16(grad_x) || !aligned16(grad_recv_x)) return EP_ERR_INVALID_ARG;
    CombineParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.expert_out = grad_recv_x;
    p.expert_out_rows = grad_recv_rows;
    p.row_of = handle->row_of;
    p.topk_weights = nullptr;  // every weight 1: the plain sum of the token's rows
    p.y = grad_x;
    p.grad_recv_w = grad_recv_topk_weights;
    p.grad_w = grad_topk_weights;
    p.status = carve_workspace(workspace, 0, 1).status;
    return cuda_status(launch_combine(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_combine_backward(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                              const void* grad_y, const void* expert_out, int64_t expert_out_rows,
                              const ep_layout* handle, const float* topk_weights,
                              void* grad_expert_out, float* grad_topk_weights, void* workspace,
                              size_t workspace_bytes, void* stream) {
    if (num_tokens < 0 || num_topk < 1 || num_topk > 32 || expert_out_rows < 0) return EP_ERR_SHAPE;
    if (num_tokens * static_cast<int64_t>(num_topk) >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    ep_status st = check_hidden(hidden, false);
    if (st != EP_OK) return st;
    if (!handle || !workspace || !aligned16(workspace) || workspace_bytes < kWsHeader)
        return EP_ERR_INVALID_ARG;
    if (num_tokens == 0) return EP_OK;
    if (!handle->row_of || !grad_y || !topk_weights || !grad_topk_weights ||
        (expert_out_rows > 0 && (!expert_out || !grad_expert_out)))
        return EP_ERR_INVALID_ARG;
    if (!aligned16(grad_y) || !aligned16(expert_out) || !aligned16(grad_expert_out))
        return EP_ERR_INVALID_ARG;
    CombineBackwardParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.grad_y = grad_y;
    p.expert_out = expert_out;
    p.expert_out_rows = expert_out_rows;
    p.row_of = handle->row_of;
    p.topk_weights = topk_weights;
    p.grad_expert_out = grad_expert_out;
    p.grad_topk_weights = grad_topk_weights;
    p.status = carve_workspace(workspace, 0, 1).status;
    return cuda_status(launch_combine_backward(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_low_latency_dispatch(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                  int32_t num_experts, int32_t num_max_tokens, const void* x,
                                  const int64_t* topk_idx, void* recv_x, float* recv_scales,
                                  int32_t* recv_expert_count, const ep_ll_handle* handle,
                                  void* workspace, size_t workspace_bytes, void* stream) {
    ep_status st = check_routing(num_tokens, num_topk, num_experts, 1);
    if (st != EP_OK) return st;
    if ((st = check_hidden(hidden, true)) != EP_OK) return st;
    if (num_max_tokens < 1 || num_tokens > num_max_tokens) return EP_ERR_SHAPE;
    if (static_cast<int64_t>(num_experts) * num_max_tokens >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    if (!handle || !workspace || !recv_expert_count || workspace_bytes < kWsHeader)
        return EP_ERR_INVALID_ARG;
    if (num_tokens > 0) {
        if (!x || !topk_idx || !recv_x || !recv_scales || !handle->row_of || !handle->src_of)
            return EP_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(recv_x) || !aligned16(recv_scales))
            return EP_ERR_INVALID_ARG;
    }
    LowLatencyDispatchParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.E = num_experts;
    p.cap = num_max_tokens;
    p.x = x;
    p.topk_idx = topk_idx;
    p.recv_x = recv_x;
    p.recv_scales = recv_scales;
    p.recv_expert_count = recv_expert_count;
    p.row_of = handle->row_of;
    p.src_of = handle->src_of;
    p.status = carve_workspace(workspace, 0, 1).status;
    p.timeout_ns = kDefaultTimeoutNs;
    return cuda_status(launch_ll_dispatch(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_low_latency_combine(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                 int32_t num_experts, int32_t num_max_tokens,
                                 const void* expert_out, const ep_ll_handle* handle,
                                 const float* topk_weights, void* y, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    if (num_experts < 1 || num_max_tokens < 1) return EP_ERR_SHAPE;
    if (!handle) return EP_ERR_INVALID_ARG;
    ep_layout lay = {};
    lay.row_of = handle->row_of;
    return ep_combine(num_tokens, hidden, num_topk, expert_out,
                      static_cast<int64_t>(num_experts) * num_max_tokens, &lay, topk_weights, y,
                      workspace, workspace_bytes, stream);
}

ep_status ep_lb_prefetch_weights(int32_t num_slots, int64_t bytes_per_slot,
                                 const int32_t* primary_of, void* weights, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    if (num_slots < 1 || num_slots > 4096 || bytes_per_slot <= 0 || bytes_per_slot % 16 != 0)
        return EP_ERR_SHAPE;
    if (!primary_of || !weights || !aligned16(weights) || !workspace ||
        workspace_bytes < kWsHeader)
        return EP_ERR_INVALID_ARG;
    const Workspace ws = carve_workspace(workspace, 0, 1);
    return cuda_status(launch_lb_prefetch(num_slots, bytes_per_slot, primary_of, weights, ws.status,
                                          static_cast<cudaStream_t>(stream)));
}

ep_status ep_lb_reduce_grads(int32_t num_slots, int64_t n, const int32_t* primary_of, float* grads,
                             void* workspace, size_t workspace_bytes, void* stream) {
    if (num_slots < 1 || num_slots > 4096 || n < 0 || n % 4 != 0) return EP_ERR_SHAPE;
    if (!primary_of || !workspace || workspace_bytes < kWsHeader) return EP_ERR_INVALID_ARG;
    if (n > 0 && (!grads || !aligned16(grads))) return EP_ERR_INVALID_ARG;
    if (n == 0) return EP_OK;
    const Workspace ws = carve_workspace(workspace, 0, 1);
    return cuda_status(launch_lb_reduce(num_slots, n, primary_of, grads, ws.status,
                                        static_cast<cudaStream_t>(stream)));
}

ep_status ep_ipc_alloc(size_t bytes, void** ptr, void* handle) {
    static_assert(sizeof(cudaIpcMemHandle_t) == EP_IPC_HANDLE_BYTES, "IPC handle size");
    if (!ptr || !handle || bytes == 0) return EP_ERR_INVALID_ARG;
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) return EP_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, p) != cudaSuccess) {
        cudaFree(p);
        return EP_ERR_CUDA;
    }
    memcpy(handle, &h, sizeof(h));
    *ptr = p;
    return EP_OK;
}

ep_status ep_ipc_free(void* ptr) {
    if (!ptr) return EP_ERR_INVALID_ARG;
    return cuda_status(cudaFree(ptr));
}

ep_status ep_ipc_open(const void* handle, void** ptr) {
    if (!handle || !ptr) return EP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof(h));
    void* p = nullptr;
    if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
        return EP_ERR_CUDA;
    *ptr = p;
    return EP_OK;
}

ep_status ep_ipc_close(void* ptr) {
    if (!ptr) return EP_ERR_INVALID_ARG;
    return cuda_status(cudaIpcCloseMemHandle(ptr));
}

ep_status ep_peer_plan(int32_t world, int32_t rank, int32_t num_experts, const int32_t* counts,
                       const int32_t* expert_offset, int64_t capacity, int32_t* dst_offset,
                       int32_t* recv_count, int32_t* recv_offset, void* workspace,
                       size_t workspace_bytes, void* stream) {
    if (world < 1 || world > 64 || num_experts < 1 || num_experts > 4096 ||
        num_experts % world != 0 || rank < 0 || rank >= world || capacity < 0 ||
        capacity >= (int64_t(1) << 31))
        return EP_ERR_SHAPE;
    if (!counts || !expert_offset || !dst_offset || !recv_count || !recv_offset || !workspace ||
        workspace_bytes < kWsHeader)
        return EP_ERR_INVALID_ARG;
    PeerPlanParams p;
    p.world = world;
    p.rank = rank;
    p.num_experts = num_experts;
    p.counts = counts;
    p.expert_offset = expert_offset;
    p.capacity = capacity;
    p.dst_offset = dst_offset;
    p.recv_count = recv_count;
    p.recv_offset = recv_offset;
    p.status = carve_workspace(workspace, 0, 1).status;
    return cuda_status(launch_peer_plan(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_peer_dispatch(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                           int32_t num_experts, int32_t world, int32_t quant, const void* x,
                           const int64_t* topk_idx, const float* topk_weights,
                           const ep_layout* handle, const int32_t* dst_offset,
                           const ep_peer_buffers* peers, void* workspace, size_t workspace_bytes,
                           void* stream) {
    if (quant != EP_QUANT_NONE && quant != EP_QUANT_FP8_E4M3_1X128 &&
        quant != EP_QUANT_FP8_E4M3_1X128_POW2)
        return EP_ERR_INVALID_ARG;  // block-major scales are not offered here
    const bool fp8 = quant != EP_QUANT_NONE;
    ep_status st = check_routing(num_tokens, num_topk, num_experts, world);
    if (st != EP_OK) return st;
    if ((st = check_hidden(hidden, fp8)) != EP_OK) return st;
    if (!peers || peers->capacity < 0 || peers->capacity >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    if (!handle || !workspace || !aligned16(workspace) || workspace_bytes < kWsHeader)
        return EP_ERR_INVALID_ARG;
    if (num_tokens == 0) return EP_OK;
    if (!handle->row_of || !x || !topk_idx || !topk_weights || !dst_offset || !peers->recv_x ||
        !peers->recv_topk_idx || !peers->recv_topk_weights || (fp8 && !peers->recv_scales) ||
        !aligned16(x))
        return EP_ERR_INVALID_ARG;
    const Workspace ws = carve_workspace(workspace, 0, 1);
    DispatchParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.slots = num_topk;
    p.dedup = 0;
    p.pow2_scales = quant == EP_QUANT_FP8_E4M3_1X128_POW2 ? 1 : 0;
    p.scales_mn = 0;
    p.scales_ld = 0;
    p.num_experts = num_experts;
    p.experts_per_partition = num_experts / world;
    p.x = x;
    p.topk_idx = topk_idx;
    p.topk_weights = topk_weights;
    p.row_of = handle->row_of;
    p.recv_x = nullptr;
    p.recv_scales = nullptr;
    p.recv_topk_idx = nullptr;
    p.recv_topk_weights = nullptr;
    p.status = ws.status;
    p.ticket = ws.ticket;
    p.done = ws.done;
    p.timeout_ns = kDefaultTimeoutNs;
    p.peer_recv_x = peers->recv_x;
    p.peer_recv_scales = fp8 ? peers->recv_scales : nullptr;
    p.peer_recv_topk_idx = peers->recv_topk_idx;
    p.peer_recv_topk_weights = peers->recv_topk_weights;
    p.peer_offset = dst_offset;
    p.peer_rows = peers->capacity;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return cuda_status(fp8 ? launch_dispatch_fp8(p, s) : launch_dispatch_bf16(p, s));
}

ep_status ep_peer_combine(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                          int32_t num_experts, int32_t world, const void* const* expert_out,
                          int64_t capacity, const ep_layout* handle, const int64_t* topk_idx,
                          const int32_t* dst_offset, const float* topk_weights, void* y,
                          void* workspace, size_t workspace_bytes, void* stream) {
    ep_status st = check_routing(num_tokens, num_topk, num_experts, world);
    if (st != EP_OK) return st;
    if ((st = check_hidden(hidden, false)) != EP_OK) return st;
    if (capacity < 0 || capacity >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    if (!handle || !workspace || workspace_bytes < kWsHeader) return EP_ERR_INVALID_ARG;
    if (num_tokens == 0) return EP_OK;
    if (!handle->row_of || !expert_out || !topk_idx || !dst_offset || !topk_weights || !y ||
        !aligned16(y))
        return EP_ERR_INVALID_ARG;
    CombineParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.expert_out = nullptr;
    p.expert_out_rows = capacity;
    p.row_of = handle->row_of;
    p.topk_weights = topk_weights;
    p.y = y;
    p.grad_recv_w = nullptr;
    p.grad_w = nullptr;
    p.status = carve_workspace(workspace, 0, 1).status;
    p.peer_out = expert_out;
    p.topk_idx = topk_idx;
    p.peer_offset = dst_offset;
    p.experts_per_partition = num_experts / world;
    p.num_experts = num_experts;
    return cuda_status(launch_combine(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_get_dispatch_layout_dedup(int64_t num_tokens, int32_t num_topk, int32_t num_experts,
                                       int32_t num_partitions, const int64_t* topk_idx,
                                       const ep_layout* layout, void* workspace,
                                       size_t workspace_bytes, void* stream) {
    ep_status st = check_routing(num_tokens, num_topk, num_experts, num_partitions);
    if (st != EP_OK) return st;
    if (num_partitions > 32) return EP_ERR_SHAPE;
    if (num_tokens * static_cast<int64_t>(num_partitions) >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    if ((st = check_layout_ptrs(layout, num_tokens)) != EP_OK) return st;
    if (!workspace || !aligned16(workspace) || (num_tokens > 0 && !topk_idx))
        return EP_ERR_INVALID_ARG;
    if (workspace_bytes < ep_workspace_bytes(num_tokens, num_experts, num_partitions))
        return EP_ERR_WORKSPACE;
    if ((st = check_layout_size(num_tokens, num_topk, num_experts, num_partitions, true)) != EP_OK)
        return st;
    const Workspace ws = carve_workspace(workspace, num_tokens, num_partitions);
    return cuda_status(launch_layout(num_tokens, num_topk, num_experts, num_partitions, topk_idx,
                                     *layout, ws, static_cast<cudaStream_t>(stream),
                                     /*by_partition=*/true));
}

ep_status ep_peer_dispatch_dedup(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                 int32_t num_experts, int32_t world, int32_t quant, const void* x,
                                 const int64_t* topk_idx, const float* topk_weights,
                                 const ep_layout* handle, const int32_t* dst_offset,
                                 const ep_peer_buffers* peers, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    if (quant != EP_QUANT_NONE && quant != EP_QUANT_FP8_E4M3_1X128 &&
        quant != EP_QUANT_FP8_E4M3_1X128_POW2)
        return EP_ERR_INVALID_ARG;
    const bool fp8 = quant != EP_QUANT_NONE;
    ep_status st = check_routing(num_tokens, num_topk, num_experts, world);
    if (st != EP_OK) return st;
    if (world > 32) return EP_ERR_SHAPE;  // one storer lane per rank
    if ((st = check_hidden(hidden, fp8)) != EP_OK) return st;
    if (!peers || peers->capacity < 0 || peers->capacity >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    if (!handle || !workspace || !aligned16(workspace) || workspace_bytes < kWsHeader)
        return EP_ERR_INVALID_ARG;
    if (num_tokens == 0) return EP_OK;
    if (!handle->row_of || !x || !topk_idx || !topk_weights || !dst_offset || !peers->recv_x ||
        !peers->recv_topk_idx || !peers->recv_topk_weights || (fp8 && !peers->recv_scales) ||
        !aligned16(x))
        return EP_ERR_INVALID_ARG;
    const Workspace ws = carve_workspace(workspace, 0, 1);
    DispatchParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.slots = world;
    p.dedup = 1;
    p.pow2_scales = quant == EP_QUANT_FP8_E4M3_1X128_POW2 ? 1 : 0;
    p.scales_mn = 0;
    p.scales_ld = 0;
    p.num_experts = num_experts;
    p.experts_per_partition = num_experts / world;
    p.x = x;
    p.topk_idx = topk_idx;
    p.topk_weights = topk_weights;
    p.row_of = handle->row_of;
    p.recv_x = nullptr;
    p.recv_scales = nullptr;
    p.recv_topk_idx = nullptr;
    p.recv_topk_weights = nullptr;
    p.status = ws.status;
    p.ticket = ws.ticket;
    p.done = ws.done;
    p.timeout_ns = kDefaultTimeoutNs;
    p.peer_recv_x = peers->recv_x;
    p.peer_recv_scales = fp8 ? peers->recv_scales : nullptr;
    p.peer_recv_topk_idx = peers->recv_topk_idx;
    p.peer_recv_topk_weights = peers->recv_topk_weights;
    p.peer_offset = dst_offset;
    p.peer_rows = peers->capacity;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return cuda_status(fp8 ? launch_dispatch_fp8(p, s) : launch_dispatch_bf16(p, s));
}

ep_status ep_peer_combine_dedup(int64_t num_tokens, int64_t hidden, int32_t world,
                                const void* const* partition_out, int64_t capacity,
                                const ep_layout* handle, const int32_t* dst_offset, void* y,
                                void* workspace, size_t workspace_bytes, void* stream) {
    if (num_tokens < 0 || world < 1 || world > 32 || capacity < 0 ||
        capacity >= (int64_t(1) << 31))
        return EP_ERR_SHAPE;
    if (num_tokens * static_cast<int64_t>(world) >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    ep_status st = check_hidden(hidden, false);
    if (st != EP_OK) return st;
    if (!handle || !workspace || workspace_bytes < kWsHeader) return EP_ERR_INVALID_ARG;
    if (num_tokens == 0) return EP_OK;
    if (!handle->row_of || !partition_out || !dst_offset || !y || !aligned16(y))
        return EP_ERR_INVALID_ARG;
    CombineParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = world;  // slots are ranks
    p.expert_out = nullptr;
    p.expert_out_rows = capacity;
    p.row_of = handle->row_of;
    p.topk_weights = nullptr;  // partitions return weighted rows: a plain sum
    p.y = y;
    p.grad_recv_w = nullptr;
    p.grad_w = nullptr;
    p.status = carve_workspace(workspace, 0, 1).status;
    p.sparse = 1;
    p.peer_out = partition_out;
    p.topk_idx = nullptr;
    p.peer_offset = dst_offset;
    p.experts_per_partition = 1;
    p.num_experts = world;
    p.peer_by_slot = 1;
    return cuda_status(launch_combine(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_peer_low_latency_dispatch(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                       int32_t num_experts, int32_t world, int32_t rank,
                                       int32_t num_max_tokens, const void* x,
                                       const int64_t* topk_idx, void* const* recv_x,
                                       float* const* recv_scales, int32_t* const* recv_expert_count,
                                       const ep_ll_handle* handle, void* workspace,
                                       size_t workspace_bytes, void* stream) {
    ep_status st = check_routing(num_tokens, num_topk, num_experts, world);
    if (st != EP_OK) return st;
    if ((st = check_hidden(hidden, true)) != EP_OK) return st;
    if (rank < 0 || rank >= world) return EP_ERR_SHAPE;
    if (num_max_tokens < 1 || num_tokens > num_max_tokens) return EP_ERR_SHAPE;
    if (static_cast<int64_t>(num_experts) * num_max_tokens >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    if (!handle || !workspace || !recv_x || !recv_scales || !recv_expert_count ||
        workspace_bytes < kWsHeader)
        return EP_ERR_INVALID_ARG;
    if (num_tokens > 0 && (!x || !topk_idx || !handle->row_of || !handle->src_of || !aligned16(x)))
        return EP_ERR_INVALID_ARG;
    LowLatencyDispatchParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.E = num_experts;
    p.cap = num_max_tokens;
    p.x = x;
    p.topk_idx = topk_idx;
    p.recv_x = nullptr;
    p.recv_scales = nullptr;
    p.recv_expert_count = nullptr;
    p.row_of = handle->row_of;
    p.src_of = handle->src_of;
    p.status = carve_workspace(workspace, 0, 1).status;
    p.timeout_ns = kDefaultTimeoutNs;
    p.peer_recv_x = recv_x;
    p.peer_recv_scales = recv_scales;
    p.peer_recv_count = recv_expert_count;
    p.world = world;
    p.rank = rank;
    p.epp = num_experts / world;
    return cuda_status(launch_ll_dispatch(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_peer_low_latency_combine(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                      int32_t num_experts, int32_t world, int32_t rank,
                                      int32_t num_max_tokens, const void* const* expert_out,
                                      const int64_t* topk_idx, const ep_ll_handle* handle,
                                      const float* topk_weights, void* y, void* workspace,
                                      size_t workspace_bytes, void* stream) {
    ep_status st = check_routing(num_tokens, num_topk, num_experts, world);
    if (st != EP_OK) return st;
    if ((st = check_hidden(hidden, false)) != EP_OK) return st;
    if (rank < 0 || rank >= world || num_max_tokens < 1) return EP_ERR_SHAPE;
    if (static_cast<int64_t>(num_experts) * num_max_tokens >= (int64_t(1) << 31)) return EP_ERR_SHAPE;
    if (!handle || !workspace || workspace_bytes < kWsHeader) return EP_ERR_INVALID_ARG;
    if (num_tokens == 0) return EP_OK;
    if (!handle->row_of || !expert_out || !topk_idx || !topk_weights || !y || !aligned16(y))
        return EP_ERR_INVALID_ARG;
    CombineParams p;
    p.T = num_tokens;
    p.H = hidden;
    p.K = num_topk;
    p.expert_out = nullptr;
    p.expert_out_rows = static_cast<int64_t>(num_experts / world) * world * num_max_tokens;
    p.row_of = handle->row_of;
    p.topk_weights = topk_weights;
    p.y = y;
    p.grad_recv_w = nullptr;
    p.grad_w = nullptr;
    p.status = carve_workspace(workspace, 0, 1).status;
    p.peer_out = expert_out;
    p.topk_idx = topk_idx;
    p.peer_offset = nullptr;
    p.experts_per_partition = num_experts / world;
    p.num_experts = num_experts;
    p.peer_ll_cap = num_max_tokens;
    p.peer_world = world;
    p.peer_rank = rank;
    return cuda_status(launch_combine(p, static_cast<cudaStream_t>(stream)));
}

ep_status ep_debug_wait_probe(uint64_t timeout_ns, void* workspace, size_t workspace_bytes,
                              void* stream) {
    if (!workspace || workspace_bytes < kWsHeader) return EP_ERR_INVALID_ARG;
    const Workspace ws = carve_workspace(workspace, 0, 1);
    return cuda_status(
        launch_wait_probe(ws.status, ws.probe_flag, timeout_ns, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
