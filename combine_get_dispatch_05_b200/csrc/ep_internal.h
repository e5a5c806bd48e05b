// ep_internal.h -- host-side launchers behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep_b200.h"

namespace ep {

// Per-device facts the launchers size grids with.
struct DeviceInfo {
    int device;
    int num_sms;
    size_t max_smem_optin;   // per CTA
    size_t smem_per_sm;      // per SM
    size_t smem_reserved;    // reserved by the runtime per resident CTA
};
cudaError_t device_info(DeviceInfo* out);

// Resident CTAs per SM (at least 1) of `kernel` launched with `threads` threads and
// `smem` bytes of dynamic shared memory on device `device`.  The answer depends
// only on the kernel and the device, so each is computed once and kept.
int blocks_per_sm(const void* kernel, int device, int threads, size_t smem);

// Host-side argument checks of the layout entry points (the workspace and the
// no-workspace forms validate alike).  check_routing: sizes in range
// (EP_ERR_SHAPE); check_layout_ptrs: the arrays a batch of T tokens needs are set
// (EP_ERR_INVALID_ARG); check_layout_size: the batch fits the layout kernel's
// shared memory (EP_ERR_SHAPE; EP_ERR_CUDA if the device cannot be queried).
ep_status check_routing(int64_t T, int32_t K, int32_t E, int32_t P);
ep_status check_layout_ptrs(const ep_layout* lay, int64_t T);
ep_status check_layout_size(int64_t T, int32_t K, int32_t E, int32_t P, bool by_partition);

// Upper bound on the layout kernel's CTAs (chunks) for a batch of num_tokens.
int64_t max_layout_chunks(int64_t num_tokens);

struct Workspace {
    uint32_t* status;
    uint32_t* probe_flag;
    unsigned long long* bar;
    int32_t* ticket;           // next token a dispatch CTA takes
    uint32_t* done;            // dispatch CTAs finished
    int32_t* chunk_expert;     // [chunks][E]
    int32_t* chunk_partition;  // [chunks][P]
};
Workspace carve_workspace(void* ws, int64_t num_tokens, int32_t num_experts);

// Launch the (cooperative) layout kernel on `stream`.  It waits for all earlier
// work in the stream and lets the next kernel start early (programmatic
// dependent launch).
// by_partition: the deduplicated layout (one slot per partition, rows
// partition-major); the layout arrays are then P-sized and row_of is [T, P].
// Whether the layout of a batch of T tokens fits the layout kernels (each SM keeps
// its chunk of ids in shared memory): *fits = false above about 400k tokens at
// K = 8, E = 256.  Returns a CUDA error only if the device cannot be queried.
cudaError_t layout_fits(int64_t T, int32_t K, int32_t E, int32_t P, bool by_partition, bool* fits);

cudaError_t launch_layout(int64_t T, int32_t K, int32_t E, int32_t P, const int64_t* topk_idx,
                          const ep_layout& lay, const Workspace& ws, cudaStream_t stream,
                          bool by_partition = false);

struct DispatchParams {
    int64_t T;
    int64_t H;
    int32_t K;       // routing ids per token (topk_idx / topk_weights row length)
    int32_t slots;   // receive rows per token in row_of: K, or P when dedup
    int32_t dedup;   // 1: a row per (token, partition) with [rows, K] expert lists
    int32_t pow2_scales;  // FP8: power-of-two block scales
    int32_t scales_mn;    // FP8: recv_scales block-major, [H/128][scales_ld]
    int64_t scales_ld;
    int32_t in_stages;    // FP8: input ring depth (rows in flight from HBM per CTA)
    int32_t out_stages;   // FP8: quantised rows staged per CTA
    int32_t num_experts;
    int32_t experts_per_partition;
    const void* x;
    const int64_t* topk_idx;
    const float* topk_weights;
    const int32_t* row_of;
    void* recv_x;
    float* recv_scales;
    int32_t* recv_topk_idx;
    float* recv_topk_weights;
    uint32_t* status;
    int32_t* ticket;  // token counter (zero on entry; the last CTA to finish re-zeroes it)
    uint32_t* done;
    uint64_t timeout_ns;
    // Peer mode (partitions are ranks): the row of (t, k) is row_of[t, k] +
    // peer_offset[e] in the buffers of rank e / experts_per_partition (deduplicated
    // rows: the row of (t, q) is row_of[t, q] + peer_offset[q] in rank q's), whose
    // base pointers the tables hold; recv_x .. recv_topk_weights are unused.
    void* const* peer_recv_x = nullptr;
    float* const* peer_recv_scales = nullptr;
    int32_t* const* peer_recv_topk_idx = nullptr;
    float* const* peer_recv_topk_weights = nullptr;
    const int32_t* peer_offset = nullptr;  // [E]; NULL: one local buffer
    int64_t peer_rows = 0;                 // rows of every rank's receive buffers
};
// Launched programmatically dependent on the preceding layout kernel.
cudaError_t launch_dispatch_fp8(const DispatchParams& p, cudaStream_t stream);
cudaError_t launch_dispatch_bf16(const DispatchParams& p, cudaStream_t stream);

struct CombineParams {
    int64_t T;
    int64_t H;
    int32_t K;
    const void* expert_out;
    int64_t expert_out_rows;
    const int32_t* row_of;
    const float* topk_weights;  // NULL: every weight is 1 (the backward of dispatch)
    void* y;
    const float* grad_recv_w;   // optional gather: grad_w[t, k] = grad_recv_w[row_of[t, k]]
    float* grad_w;
    uint32_t* status;
    int32_t sparse = 0;         // about half the slots empty (one slot per partition)
    // Peer mode (partitions are ranks): the row of (t, k) is row_of[t, k] +
    // peer_offset[e], e = topk_idx[t, k], in peer_out[e / experts_per_partition];
    // expert_out is unused and expert_out_rows bounds every rank's rows.
    const void* const* peer_out = nullptr;
    const int64_t* topk_idx = nullptr;
    const int32_t* peer_offset = nullptr;
    int32_t experts_per_partition = 1;
    int32_t num_experts = 0;
    int32_t peer_by_slot = 0;  // deduplicated rows: slot k is rank k (topk_idx unused)
    // low-latency rows (row_of = e * cap + j): the row is ((e % epp) * peer_world +
    // peer_rank) * peer_ll_cap + j in rank e / epp's outputs (peer_offset unused)
    int32_t peer_ll_cap = 0, peer_world = 1, peer_rank = 0;
};
cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream);

// Destination offsets of one rank's rows in the owners' receive buffers, from every
// rank's per-expert counts (one CTA).
struct PeerPlanParams {
    int32_t world, rank, num_experts;
    const int32_t* counts;         // [world, E]: num_tokens_per_expert of every rank
    const int32_t* expert_offset;  // [E + 1]: this rank's layout
    int64_t capacity;              // rows of every rank's receive buffers
    int32_t* dst_offset;           // [E]
    int32_t* recv_count;           // [E / world]: rows this rank receives per local expert
    int32_t* recv_offset;          // [E / world + 1]
    uint32_t* status;
};
cudaError_t launch_peer_plan(const PeerPlanParams& p, cudaStream_t stream);

struct CombineBackwardParams {
    int64_t T;
    int64_t H;
    int32_t K;
    const void* grad_y;
    const void* expert_out;
    int64_t expert_out_rows;
    const int32_t* row_of;
    const float* topk_weights;
    void* grad_expert_out;
    float* grad_topk_weights;
    uint32_t* status;
};
cudaError_t launch_combine_backward(const CombineBackwardParams& p, cudaStream_t stream);

struct LowLatencyDispatchParams {
    int64_t T;
    int64_t H;
    int32_t K;
    int32_t E;
    int32_t cap;
    const void* x;
    const int64_t* topk_idx;
    void* recv_x;
    float* recv_scales;
    int32_t* recv_expert_count;
    int32_t* row_of;
    int32_t* src_of;
    uint32_t* status;
    uint64_t timeout_ns;
    // Peer mode (partitions are the ranks of a node): slot j of expert e goes to row
    // ((e % epp) * world + rank) * cap + j of rank e / epp's buffers, and the count of
    // e to entry (e % epp) * world + rank of its count table; recv_x, recv_scales and
    // recv_expert_count are unused (row_of / src_of stay local: e * cap + j).
    void* const* peer_recv_x = nullptr;
    float* const* peer_recv_scales = nullptr;
    int32_t* const* peer_recv_count = nullptr;
    int32_t world = 1, rank = 0, epp = 1;
};
cudaError_t launch_ll_dispatch(const LowLatencyDispatchParams& p, cudaStream_t stream);

cudaError_t launch_lb_prefetch(int32_t S, int64_t nbytes, const int32_t* primary_of, void* weights,
                               uint32_t* status, cudaStream_t stream);
cudaError_t launch_lb_reduce(int32_t S, int64_t n, const int32_t* primary_of, float* grads,
                             uint32_t* status, cudaStream_t stream);

cudaError_t launch_wait_probe(uint32_t* status, uint32_t* flag, uint64_t timeout_ns,
                              cudaStream_t stream);

// Default bound on any device-side wait (device time).
constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;

}  // namespace ep
