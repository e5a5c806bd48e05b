// layout_static.cu -- ep_get_dispatch_layout_static: the routing layout without a
// caller-provided workspace.
//
// Some callers cannot allocate device memory where they call the layout: an
// inference engine that hands all of HBM to its own pool at start-up, a plugin
// whose enqueue step must not allocate, or a latency-critical path where the
// implicit device synchronisation of cudaMalloc would stall other streams.  This
// entry point gives them the same layout as ep_get_dispatch_layout, with its
// scratch (status word, grid-barrier words, per-chunk expert and partition counts) in
// a fixed array compiled into the library instead of a workspace.
//
// The array below is EP_STATIC_SCRATCH_BYTES (1 MiB) per GPU; every GPU that
// loads the library holds it until the process exits.  All calls share it and it
// keeps the last call's contents, so calls that overlap on the GPU (different
// streams, or different host threads on one device) race; calls in one stream
// are ordered and safe.  Nothing here allocates: no cudaMalloc, no cudaFree, no
// allocating library routine.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "ep_b200.h"
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace {

static __device__ __align__(256) uint8_t g_layout_scratch[EP_STATIC_SCRATCH_BYTES];

constexpr int kMaxStaticDevices = 64;
std::mutex g_setup_mutex;
std::atomic<int> g_ready[kMaxStaticDevices];
void* g_scratch_ptr[kMaxStaticDevices];

// Device address of g_layout_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once per
// device with that device current, and cached.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxStaticDevices) return cudaErrorInvalidDevice;
    if (g_ready[dev].load(std::memory_order_acquire)) {
        *out = g_scratch_ptr[dev];
        return cudaSuccess;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_ready[dev].load(std::memory_order_relaxed)) {
        void* ptr = nullptr;
        err = cudaGetSymbolAddress(&ptr, g_layout_scratch);
        if (err != cudaSuccess) return err;
        if (ptr == nullptr) return cudaErrorInvalidSymbol;
        g_scratch_ptr[dev] = ptr;
        g_ready[dev].store(1, std::memory_order_release);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" ep_status ep_get_dispatch_layout_static(int64_t num_tokens, int32_t num_topk,
                                                   int32_t num_experts, int32_t num_partitions,
                                                   const int64_t* topk_idx,
                                                   const ep_layout* layout, void* stream) {
    if (num_tokens < 0 || num_topk < 1 || num_topk > 32 || num_experts < 1 ||
        num_experts > 4096 || num_partitions < 1 || num_partitions > 64 ||
        num_experts % num_partitions != 0 ||
        num_tokens * static_cast<int64_t>(num_topk) >= (int64_t(1) << 31))
        return EP_ERR_SHAPE;
    if (!layout || !layout->num_tokens_per_expert || !layout->num_tokens_per_partition ||
        !layout->expert_offset || !layout->num_recv)
        return EP_ERR_INVALID_ARG;
    if (num_tokens > 0 &&
        (!topk_idx || !layout->is_token_in_partition || !layout->row_of || !layout->src_of))
        return EP_ERR_INVALID_ARG;
    // the batch must fit the built-in scratch
    if (ep_workspace_bytes(num_tokens, num_experts, num_partitions) > EP_STATIC_SCRATCH_BYTES)
        return EP_ERR_WORKSPACE;

    bool fits = true;
    if (layout_fits(num_tokens, num_topk, num_experts, num_partitions, false, &fits) != cudaSuccess)
        return EP_ERR_CUDA;
    if (!fits) return EP_ERR_SHAPE;
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return EP_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // status word and grid-barrier counter must start at zero; the per-chunk counts are
    // fully written before they are read
    if (cudaMemsetAsync(scratch, 0, kWsHeader, s) != cudaSuccess) return EP_ERR_CUDA;
    const Workspace ws = carve_workspace(scratch, num_tokens, num_experts);
    return launch_layout(num_tokens, num_topk, num_experts, num_partitions, topk_idx, *layout, ws,
                         s) == cudaSuccess
               ? EP_OK
               : EP_ERR_CUDA;
}
