// layout_static.cu -- ep_get_dispatch_layout_static: the routing layout without a
// caller-provided workspace.
//
// Some callers cannot allocate device memory where they call the layout: an
// inference engine that hands all of HBM to its own pool at start-up, a plugin
// whose enqueue step must not allocate, or a latency-critical path where the
// implicit device synchronisation of cudaMalloc would stall other streams.  This
// entry point gives them the same layout as ep_get_dispatch_layout, with its
// scratch (status word, grid-barrier word, per-chunk expert and partition counts) in
// a fixed array compiled into the library instead of a workspace.
//
// The array below is EP_STATIC_SCRATCH_BYTES (1 MiB) per GPU; every GPU that
// loads the library holds it until the process exits.  All calls share it and it
// keeps the last call's contents, so calls that overlap on the GPU (different
// streams, or different host threads on one device) race; calls in one stream
// are ordered and safe.  Nothing here allocates: no cudaMalloc, no cudaFree, no
// allocating library routine.
#include <cuda.h>  // CUcontext / CUresult types only: the driver is reached through
                   // the runtime's entry-point query, not linked
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ep_b200.h"
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace {

static __device__ __align__(256) uint8_t g_layout_scratch[EP_STATIC_SCRATCH_BYTES];

constexpr int kMaxStaticDevices = 64;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

std::mutex g_mutex;  // guards everything below
bool g_have_fns = false;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
unsigned long long g_ctx_id[kMaxStaticDevices];  // context the cached address belongs to (0: none)
void* g_scratch_ptr[kMaxStaticDevices];

// Unique id of the calling thread's current context, 0 if there is none yet.
cudaError_t current_context_id(unsigned long long* id) {
    *id = 0;
    if (!g_have_fns) {
        cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
        cudaError_t err = cudaGetDriverEntryPointByVersion(
            "cuCtxGetCurrent", reinterpret_cast<void**>(&g_ctx_get_current), 12000,
            cudaEnableDefault, &q1);
        if (err != cudaSuccess) return err;
        err = cudaGetDriverEntryPointByVersion("cuCtxGetId", reinterpret_cast<void**>(&g_ctx_get_id),
                                               12000, cudaEnableDefault, &q2);
        if (err != cudaSuccess) return err;
        if (q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess ||
            !g_ctx_get_current || !g_ctx_get_id)
            return cudaErrorNotSupported;
        g_have_fns = true;
    }
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
    if (ctx == nullptr) return cudaSuccess;
    return g_ctx_get_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorUnknown;
}

// Device address of g_layout_scratch in the current context.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with the
// device current and cached together with the id of the context it belongs to;
// a different current context (a device reset re-creates it, and the array may
// move) makes the next call look it up again.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxStaticDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    unsigned long long id = 0;
    if ((err = current_context_id(&id)) != cudaSuccess) return err;
    if (id == 0 || g_ctx_id[dev] != id) {
        void* ptr = nullptr;
        err = cudaGetSymbolAddress(&ptr, g_layout_scratch);  // makes the context current
        if (err != cudaSuccess) return err;
        if (ptr == nullptr) return cudaErrorInvalidSymbol;
        if ((err = current_context_id(&id)) != cudaSuccess) return err;
        g_scratch_ptr[dev] = ptr;
        g_ctx_id[dev] = id;
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
    // the same checks as ep_get_dispatch_layout, in the same order
    ep_status st = check_routing(num_tokens, num_topk, num_experts, num_partitions);
    if (st != EP_OK) return st;
    if ((st = check_layout_ptrs(layout, num_tokens)) != EP_OK) return st;
    if (num_tokens > 0 && !topk_idx) return EP_ERR_INVALID_ARG;
    // the batch must fit the built-in scratch
    if (ep_workspace_bytes(num_tokens, num_experts, num_partitions) > EP_STATIC_SCRATCH_BYTES)
        return EP_ERR_WORKSPACE;
    if ((st = check_layout_size(num_tokens, num_topk, num_experts, num_partitions, false)) != EP_OK)
        return st;
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
