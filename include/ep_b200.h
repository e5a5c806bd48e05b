/*
 * ep_b200.h -- C ABI of the B200 (sm_100a) MoE token dispatch / combine library.
 *
 * The library is the single-GPU hot path of an expert-parallel (EP)
 * communication layer in the style of DeepEP:
 *
 *   - layout:   from topk_idx, count rows per expert and tokens per logical
 *               partition, and give every (token, top-k slot) a stable row in an
 *               expert-contiguous receive buffer;
 *   - dispatch: quantise each token's BF16 hidden vector to FP8 (or copy it as
 *               BF16) and write it to each of its rows;
 *   - combine:  gather the expert outputs of a token's rows and reduce them,
 *               weighted by topk_weights, back into token order in BF16;
 *   - low-latency dispatch / combine: the same for small decode batches, into a
 *               padded [num_experts, num_max_tokens, hidden] receive tensor.
 *
 * Sources (the DeepEP pages):
 *   "DeepSeek 开源周第二弹：DeepEP —— 首个 MoE 模型训练和推理的 EP 通信库"
 *   (m.youleyou.com), sections "DeepEP 的核心功能" and
 *   "DeepEP 的常规内核和低延迟内核": normal kernels for training / prefill,
 *   low-latency kernels for decode, FP8 dispatch, BF16 result merge.
 *   deepseek.csdn.net/67bd3eb22e30c863900615cc, sections "使用示例 / MoE 训练中的
 *   应用" (dispatch(x, topk_idx, topk_weights, num_experts) returning recv_x,
 *   recv_topk_idx, recv_topk_weights, handle, event) and "推理解码阶段的应用"
 *   (low_latency_dispatch(hidden_states, topk_idx, num_max_tokens,
 *   num_experts) returning recv_hidden_states, recv_expert_count, handle,
 *   event, hook; buffer of num_max_tokens * hidden * num_experts elements).
 *   "deepseek-ai/DeepEP" (agentlenshq.com), section "典型工作流程": dispatch,
 *   expert GEMM, combine reduces the expert outputs back.
 *
 * On one GPU the EP "ranks" are logical partitions of one HBM buffer:
 * partition p owns experts [p*E/P, (p+1)*E/P) and, because the receive buffer
 * is expert-major, one contiguous slice of rows.  The exchange is a
 * device-local permutation; there is no inter-GPU traffic.  Across the GPUs of
 * a node (partitions = ranks, one process per GPU) the ep_peer_* calls at the
 * end of this header store the rows straight into the owner ranks' receive
 * buffers and read the expert outputs back from them (CUDA IPC mappings).
 *
 * Conventions (every entry point):
 *   - Pointers named as device memory must be device (or managed) memory of
 *     the current CUDA device.  Every buffer is owned and allocated by the
 *     caller; the library allocates nothing (except ep_ipc_alloc, on request)
 *     and keeps no state between calls apart from a per-device cache of the SM
 *     count and kernel attributes.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call is asynchronous on that stream; host-side argument checks
 *     run before anything is enqueued and return an error synchronously.
 *   - Device-side problems (an out-of-range expert id, a full low-latency
 *     expert, a bounded wait that gave up) never trap: the offending row is
 *     skipped and a sticky bit is set in the workspace's status word, read
 *     and cleared by ep_read_status().
 *   - A workspace may be used by one stream at a time; calls that share a
 *     workspace on different streams race.
 *   - Layouts: row-major, contiguous.  x / expert_out / y are BF16 bit
 *     patterns; FP8 payload is OCP E4M3 (one byte per element).  topk_idx is
 *     int64 (the dtype torch.topk returns), -1 marks a masked slot.
 *   - Sizes: T = num_tokens >= 0, K = num_topk in [1, 32], E = num_experts in
 *     [1, 4096], P = num_partitions in [1, 64] dividing E, H = hidden > 0 with
 *     H % 8 == 0 (BF16) or H % 128 == 0 (FP8), H <= 16384; T * K < 2^31.
 *     Base pointers of x, recv_x, recv_scales, expert_out, y and the workspace
 *     must be 16-byte aligned (rows move by 16-byte vectors and bulk copies;
 *     the workspace holds 64-bit atomics).
 */
#ifndef EP_B200_H
#define EP_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

/* Host-side return codes. */
typedef enum ep_status {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1, /* a required pointer is NULL, misaligned, or an enum is unknown */
    EP_ERR_SHAPE = 2,       /* a size is outside the supported range (see Conventions),
                               or a batch is too large for the layout kernels, which keep
                               each SM's chunk of ids in shared memory (about 400k tokens
                               at K = 8, E = 256) */
    EP_ERR_WORKSPACE = 3,   /* workspace smaller than ep_workspace_bytes() */
    EP_ERR_CUDA = 4         /* the CUDA runtime reported an error (launch / copy) */
} ep_status;

/* Sticky device status bits (ep_read_status). */
#define EP_DEV_INDEX_RANGE 0x1u /* an expert id outside [-1, E) or a row outside the buffer: skipped */
#define EP_DEV_TIMEOUT 0x2u     /* a bounded device wait gave up; the kernel stopped early */
#define EP_DEV_CAPACITY 0x4u    /* a low-latency row did not fit num_max_tokens, or a rank's
                                   receive buffer was too small (peer mode): dropped */

/* Dispatch payload format. */
typedef enum ep_quant {
    EP_QUANT_NONE = 0,                /* BF16 rows copied bit for bit */
    EP_QUANT_FP8_E4M3_1X128 = 1,      /* E4M3 codes + one fp32 scale per 128 channels */
    EP_QUANT_FP8_E4M3_1X128_POW2 = 2  /* the same with each scale rounded up to a power of
                                         two (an 8-bit exponent, UE8M0, for FP8 GEMMs that
                                         take exponent-only scales); x / s is exact */
} ep_quant;

/* OR-ed into an FP8 `quant` of ep_dispatch / ep_dispatch_dedup: write recv_scales
 * MN-major (block-major), the layout FP8 grouped GEMMs read with TMA: the scale
 * of row r, block b at recv_scales[b * ld + r], ld = the worst-case row count
 * (T*K, resp. T*min(P, K)) rounded up to a multiple of 4, so every block's column
 * starts on a 16-byte boundary; recv_scales then holds (H/128) * ld floats.  The
 * values are those of the row-major layout.  The pages fix no scale layout; this
 * is a reading for the downstream expert GEMM ("deepseek-ai/DeepEP", section
 * "典型工作流程": dispatch, then the expert GEMM). */
#define EP_QUANT_SCALES_MN_MAJOR 0x100

/*
 * The layout of one batch, and the `handle` that dispatch returns and combine
 * consumes (deepseek.csdn.net/67bd3eb22e30c863900615cc, "使用示例": dispatch
 * returns a handle).  A struct of caller-owned device pointers:
 *   num_tokens_per_expert[E]     rows routed to expert e
 *   num_tokens_per_partition[P]  distinct tokens that name >= 1 expert of partition p
 *   is_token_in_partition[T*P]   uint8 0/1
 *   expert_offset[E+1]           exclusive prefix sum of num_tokens_per_expert
 *   row_of[T*K]                  receive row of (t, k); -1 for a masked / skipped slot
 *   src_of[T*K]                  inverse of row_of: t*K + k for rows [0, num_recv)
 *   num_recv[1]                  R = number of receive rows
 * Row order: expert id ascending, then token ascending, then k ascending.
 */
typedef struct ep_layout {
    int32_t* num_tokens_per_expert;
    int32_t* num_tokens_per_partition;
    uint8_t* is_token_in_partition;
    int32_t* expert_offset;
    int32_t* row_of;
    int32_t* src_of;
    int32_t* num_recv;
} ep_layout;

/*
 * Handle of a low-latency dispatch (caller-owned device pointers):
 *   row_of[T*K]   e * num_max_tokens + slot, or -1 (masked, skipped or dropped)
 *   src_of[E*num_max_tokens]   t*K + k for slots [0, recv_expert_count[e]); other slots unwritten
 */
typedef struct ep_ll_handle {
    int32_t* row_of;
    int32_t* src_of;
} ep_ll_handle;

/* Version of this ABI (incremented on any signature change). */
EP_API int32_t ep_abi_version(void);

/* Human-readable name of an ep_status value. */
EP_API const char* ep_status_string(int32_t status);

/* Bytes of device workspace the calls need for a batch of num_tokens tokens
 * (status word, grid-barrier word, the dispatch kernels' token ticket counter,
 * per-chunk expert and partition counts).  The same workspace serves every entry
 * point for batches up to that size. */
EP_API size_t ep_workspace_bytes(int64_t num_tokens, int32_t num_experts, int32_t num_partitions);

/* Zero a workspace (once, after allocating it) on `stream`.  Every call leaves
 * the barrier word and the ticket counter as it found them (the last dispatch
 * CTA to finish re-zeroes the counter).  Zero it again after a call reported
 * EP_DEV_TIMEOUT: a layout that gave up at its grid barrier leaves the barrier
 * word mid-count. */
EP_API ep_status ep_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream`, return the sticky device status bits in *bits_out and
 * clear them.  The only call that blocks the host. */
EP_API ep_status ep_read_status(void* workspace, size_t workspace_bytes, void* stream, uint32_t* bits_out);

/*
 * Routing layout of topk_idx[T*K] (device, int64) into *layout (all seven
 * arrays written).  Per-expert counts, per-partition distinct-token counts and
 * flags, expert offsets, and the stable row of every (t, k).  An id outside
 * [-1, E) is treated as masked and sets EP_DEV_INDEX_RANGE.
 * Source: the `handle` that dispatch returns and combine takes back
 * (deepseek.csdn.net/67bd3eb22e30c863900615cc, "使用示例": dispatch(x,
 * topk_idx, topk_weights, num_experts) -> recv_x, recv_topk_idx,
 * recv_topk_weights, handle, event).  The pages name the handle but not its
 * contents; what it holds here -- per-expert and per-partition counts, a
 * warp-ranked prefix scan into expert offsets and a stable slot per (t, k) by
 * token index -- is this library's reading of that handle, the layout a
 * DeepEP-style dispatch needs before it can place any row.
 */
EP_API ep_status ep_get_dispatch_layout(int64_t num_tokens, int32_t num_topk, int32_t num_experts,
                                 int32_t num_partitions, const int64_t* topk_idx,
                                 const ep_layout* layout, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* Size of the scratch array compiled into the library for
 * ep_get_dispatch_layout_static (per GPU, held until the process exits). */
#define EP_STATIC_SCRATCH_BYTES (1u << 20)

/*
 * ep_get_dispatch_layout without a workspace.  The DeepEP pages have no
 * counterpart: this entry point exists for callers that cannot allocate device
 * memory where they call the layout -- an engine that gives all of HBM to its
 * own pool at start-up, a plugin whose enqueue step must not allocate, or a
 * latency-critical path where cudaMalloc's implicit synchronisation would stall
 * other streams.  It computes exactly what ep_get_dispatch_layout computes, with
 * its scratch in a fixed EP_STATIC_SCRATCH_BYTES array inside the library.
 *   - Allocates nothing (no cudaMalloc / cudaFree / allocating library call).
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Returns EP_ERR_WORKSPACE when the batch needs more scratch than the
 *     array holds, i.e. ep_workspace_bytes(T, E, P) > EP_STATIC_SCRATCH_BYTES
 *     (about 125k tokens at E = 256, P = 8).
 *   - Every call shares the one array and it keeps the last call's contents:
 *     each call clears the part that must start at zero, and calls that overlap
 *     on the GPU (other streams or host threads on the same device) race.
 *   - Ids outside [-1, E) are skipped as masked.  This variant keeps its status
 *     word inside the private array, so nothing it would report reaches the
 *     caller: neither such ids nor a grid barrier that gave up after its bounded
 *     wait (a layout that then stops early, leaving row_of partly written).
 *     Callers that must see either use ep_get_dispatch_layout and
 *     ep_read_status.
 *   - The cached address belongs to the CUDA context current at the first
 *     call; it is looked up again whenever the device's current context
 *     changes (after cudaDeviceReset, for instance).
 */
EP_API ep_status ep_get_dispatch_layout_static(int64_t num_tokens, int32_t num_topk,
                                               int32_t num_experts, int32_t num_partitions,
                                               const int64_t* topk_idx, const ep_layout* layout,
                                               void* stream);

/*
 * Dispatch (deepseek.csdn.net/67bd3eb22e30c863900615cc, "使用示例":
 * dispatch(x, topk_idx, topk_weights, num_experts) -> recv_x, recv_topk_idx,
 * recv_topk_weights, handle, event).  Computes the layout into *handle, then
 * writes token t to every row row_of[t, k]:
 *   quant = EP_QUANT_FP8_E4M3_1X128: recv_x (uint8 [T*K, H]) gets E4M3 codes
 *     q = e4m3_rne_satfinite(x / s) and recv_scales (fp32 [T*K, H/128]) gets
 *     s = max(amax, 1e-4) / 448 of each 128-channel block (fp32 division);
 *   quant = EP_QUANT_FP8_E4M3_1X128_POW2: the same with every s rounded up to
 *     a power of two;
 *   quant | EP_QUANT_SCALES_MN_MAJOR (FP8 only): recv_scales block-major,
 *     [H/128, ld] with ld = T*K rounded up to 4;
 *   quant = EP_QUANT_NONE: recv_x (BF16 [T*K, H]) gets the row bit for bit;
 *     recv_scales may be NULL.
 *   recv_topk_idx[row] = e - p*E/P (expert id local to its partition, int32),
 *   recv_topk_weights[row] = topk_weights[t, k].
 * Receive buffers are sized for the worst case (T*K rows) so no host sync is
 * needed; the first *handle->num_recv rows are valid.  Which CTA writes a token
 * is decided at run time (a ticket counter in the workspace); what is written
 * is not, so the output is deterministic.
 * x: BF16 [T, H]; topk_idx: int64 [T, K]; topk_weights: fp32 [T, K] (device).
 */
EP_API ep_status ep_dispatch(int64_t num_tokens, int64_t hidden, int32_t num_topk, int32_t num_experts,
                      int32_t num_partitions, int32_t quant, const void* x, const int64_t* topk_idx,
                      const float* topk_weights, void* recv_x, float* recv_scales,
                      int32_t* recv_topk_idx, float* recv_topk_weights, const ep_layout* handle,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Combine ("DeepSeek 开源周第二弹：DeepEP", "DeepEP 的常规内核和低延迟内核": BF16
 * result merge; "deepseek-ai/DeepEP", "典型工作流程": combine reduces the
 * expert outputs back).  For every token t and channel i:
 *   acc = +0.0f; for k = 0..K-1 with row = handle->row_of[t, k] >= 0:
 *       acc = fmaf(topk_weights[t, k], float(expert_out[row, i]), acc)
 *   y[t, i] = bf16_round_to_nearest_even(acc)
 * expert_out: BF16 [expert_out_rows, H]; a row >= expert_out_rows is skipped
 * and sets EP_DEV_INDEX_RANGE.  y: BF16 [T, H].  Only handle->row_of is read.
 */
EP_API ep_status ep_combine(int64_t num_tokens, int64_t hidden, int32_t num_topk, const void* expert_out,
                     int64_t expert_out_rows, const ep_layout* handle, const float* topk_weights,
                     void* y, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Deduplicated dispatch: one receive row per (token, partition) instead of one per
 * (token, expert), as DeepEP's normal kernels send a token once to each rank that
 * holds any of its experts (deepseek.csdn.net/67bd3eb22e30c863900615cc, "使用示例":
 * recv_topk_idx / recv_topk_weights list each received token's local experts;
 * "DeepSeek 开源周第二弹：DeepEP", "DeepEP 的常规内核和低延迟内核": top-4 groups of
 * top-8 experts).  Under top-4-group routing a token reaches at most 4 of 8
 * partitions, so this writes at most half the rows of ep_dispatch.
 * The handle's arrays are partition-sized: num_tokens_per_expert[P] = rows per
 * partition, expert_offset[P+1], row_of[T, P] (-1 where the token names no
 * expert of the partition), src_of[rows] = t*P + p, num_recv; plus the usual
 * is_token_in_partition / num_tokens_per_partition.  Rows are partition-major,
 * token ascending.  Payload as ep_dispatch.  recv_topk_idx / recv_topk_weights
 * are [rows, K]: entry k of token t's row in partition p holds e - p*E/P and
 * topk_weights[t, k] if e = topk_idx[t, k] lies in p, else -1 and 0.
 * Receive buffers: worst case T * min(P, K) rows.  Requires P <= 32.
 */
EP_API ep_status ep_dispatch_dedup(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                   int32_t num_experts, int32_t num_partitions, int32_t quant,
                                   const void* x, const int64_t* topk_idx,
                                   const float* topk_weights, void* recv_x, float* recv_scales,
                                   int32_t* recv_topk_idx, float* recv_topk_weights,
                                   const ep_layout* handle, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * Combine of the deduplicated path: each partition returns one row per received
 * token, already reduced over its own experts with their weights, so
 *   y[t, i] = bf16_rne( (+0.0f + out[row_of[t,0], i]) + out[row_of[t,1], i] + ... )
 * over the token's partitions in partition order (fp32 adds).
 * partition_out: BF16 [partition_out_rows, H]; row_of from ep_dispatch_dedup's handle.
 */
EP_API ep_status ep_combine_dedup(int64_t num_tokens, int64_t hidden, int32_t num_partitions,
                                  const void* partition_out, int64_t partition_out_rows,
                                  const ep_layout* handle, void* y, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * Backward of dispatch ("deepseek-ai/DeepEP" (agentlenshq.com), section
 * "典型工作流程": combine or the backward helpers reduce results back).  Each
 * receive row is a copy of its token, so the gradient of x is the plain sum of
 * the gradients of the token's rows:
 *   grad_x[t, i] = bf16_rne( ((+0.0f + g[row_of[t,0], i]) + g[row_of[t,1], i]) + ... )
 * over valid slots in k order (fp32 adds), g = grad_recv_x BF16 [grad_recv_rows, H];
 * and, if both pointers are given (else both NULL),
 *   grad_topk_weights[t, k] = grad_recv_topk_weights[row_of[t, k]] (0 for masked slots).
 * grad_x: BF16 [T, H].  Only handle->row_of is read.
 */
EP_API ep_status ep_dispatch_backward(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                      const void* grad_recv_x, int64_t grad_recv_rows,
                                      const ep_layout* handle, const float* grad_recv_topk_weights,
                                      void* grad_x, float* grad_topk_weights, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * Backward of combine (y[t] = sum_k w[t,k] * expert_out[row_of[t,k]]):
 *   grad_expert_out[row_of[t,k], i] = bf16_rne( w[t,k] * float(grad_y[t, i]) )  (fp32 multiply)
 *   grad_topk_weights[t, k] = float( sum_i (double)grad_y[t,i] * (double)expert_out[row,i] ),
 *                             0 for masked slots.
 * BF16 products are exact in fp32 and the sum runs in fp64, which is exact (so
 * order-independent) while the products span fewer than 37 binades.  Rows that
 * no slot points at are not written; each row must be named by at most one slot
 * (true of every layout this library produces).  grad_y, expert_out,
 * grad_expert_out: BF16; grad_topk_weights: fp32 [T, K].
 */
EP_API ep_status ep_combine_backward(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                     const void* grad_y, const void* expert_out,
                                     int64_t expert_out_rows, const ep_layout* handle,
                                     const float* topk_weights, void* grad_expert_out,
                                     float* grad_topk_weights, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * Low-latency dispatch (deepseek.csdn.net/67bd3eb22e30c863900615cc,
 * "推理解码阶段的应用").  One fused kernel: layout, FP8 quantisation and
 * scatter into the padded tensors
 *   recv_x      uint8 [E, num_max_tokens, H]      (E4M3 codes)
 *   recv_scales fp32  [E, num_max_tokens, H/128]
 * Slot j of (t, k) inside expert e is its rank among e's rows in
 * (token, k) order -- the same order as the normal layout, so slot j of
 * expert e holds normal row expert_offset[e] + j.  recv_expert_count[E]
 * (int32) = rows written per expert.  Requires T <= num_max_tokens; a row at
 * slot >= num_max_tokens (possible only when a token names an expert twice)
 * is dropped and sets EP_DEV_CAPACITY.  Unused slots are not written.
 */
EP_API ep_status ep_low_latency_dispatch(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                  int32_t num_experts, int32_t num_max_tokens, const void* x,
                                  const int64_t* topk_idx, void* recv_x, float* recv_scales,
                                  int32_t* recv_expert_count, const ep_ll_handle* handle,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * Low-latency combine ("DeepSeek 开源周第二弹：DeepEP", "DeepEP 的常规内核和低延迟
 * 内核": the low-latency kernels serve decode with FP8 dispatch and BF16 result
 * merge): the combine reduce above, with the same fixed k order and fp32 fmaf
 * chain, over expert_out BF16 [E, num_max_tokens, H] addressed by
 * handle->row_of (row e * num_max_tokens + slot).  Only handle->row_of is read;
 * a row outside [0, E * num_max_tokens) is skipped and sets EP_DEV_INDEX_RANGE.
 * y: BF16 [T, H].  Errors as for ep_combine.
 */
EP_API ep_status ep_low_latency_combine(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                 int32_t num_experts, int32_t num_max_tokens,
                                 const void* expert_out, const ep_ll_handle* handle,
                                 const float* topk_weights, void* y, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * Test hook for the bounded device waits: launches one tiny kernel that waits
 * on a workspace flag nothing sets and on an mbarrier transaction nothing
 * completes, each for at most timeout_ns; both give up, set EP_DEV_TIMEOUT and
 * return, leaving the context usable.
 */
EP_API ep_status ep_debug_wait_probe(uint64_t timeout_ns, void* workspace, size_t workspace_bytes,
                              void* stream);

/* ---- redundant experts ----------------------------------------------------
 * "deepseek-ai/DeepEP" (agentlenshq.com), section "主要特性" (redundant-expert
 * support: lb_prefetch_weights / lb_reduce_grads) and section "典型工作流程",
 * step 5 (optionally replicate heavily loaded experts across NVLink-connected
 * GPUs).  The pages name the calls and their purpose; this library's reading on
 * one GPU, whose expert slots stand for the ranks' slots:
 *   primary_of  device int32 [num_slots]: the slot holding slot s's
 *               authoritative copy (a primary names itself, a replica its
 *               primary).  An entry out of [0, num_slots) or naming a slot that
 *               is not a primary is skipped and sets EP_DEV_INDEX_RANGE.
 * Asynchronous on `stream`; the workspace carries the status word only
 * (workspace_bytes >= 256 suffices).  Errors: EP_ERR_INVALID_ARG for NULL or
 * misaligned pointers, EP_ERR_SHAPE for sizes out of range. */

/* Copy every primary's weight blob into its replica slots.
 *   weights  device, 16-byte aligned, [num_slots, bytes_per_slot] bytes;
 *            primaries are read, replicas written.
 *   bytes_per_slot > 0, a multiple of 16; 1 <= num_slots <= 4096. */
EP_API ep_status ep_lb_prefetch_weights(int32_t num_slots, int64_t bytes_per_slot,
                                        const int32_t* primary_of, void* weights, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Sum the fp32 gradients of each primary and its replicas in ascending slot order
 * (the first member's value, then one IEEE binary32 add per further member) and
 * write the sum to every member, so all copies apply the same update.  Groups of
 * one are left untouched.
 *   grads  device, 16-byte aligned, float32 [num_slots, n], updated in place.
 *   n >= 0, a multiple of 4; 1 <= num_slots <= 4096. */
EP_API ep_status ep_lb_reduce_grads(int32_t num_slots, int64_t n, const int32_t* primary_of,
                                    float* grads, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* ---- expert parallelism across GPUs (partitions are ranks) ------------------
 * "DeepSeek 开源周第二弹：DeepEP", section "DeepEP 的常规内核和低延迟内核": the
 * normal kernels move tokens between the GPUs of a node over NVLink;
 * "deepseek-ai/DeepEP", section "典型工作流程": dispatch to the ranks that hold the
 * experts, expert computation, combine back to where the tokens came from.
 *
 * With W ranks (one process per GPU), rank p owns experts [p*E/W, (p+1)*E/W).
 * Every rank maps every rank's receive buffers (CUDA IPC, ep_ipc_*), and the
 * dispatch kernel stores each row straight into its owner's buffer; the combine
 * kernel reads the expert outputs straight from the owners' buffers.  Rank p's
 * receive rows are ordered expert (ascending), then source rank, then source
 * (token, k): exactly partition p's rows of the one-GPU dispatch of all ranks'
 * tokens concatenated in rank order.  One step on rank s:
 *   1. ep_get_dispatch_layout with num_partitions = W (handle, per-expert counts);
 *   2. the caller gathers every rank's num_tokens_per_expert into counts[W, E]
 *      (e.g. an all-gather; a few KB);
 *   3. ep_peer_plan: destination offsets of this rank's rows, and this rank's
 *      receive counts / offsets;
 *   4. the caller makes sure every rank is past its use of the buffers this step
 *      overwrites (step 2's collective does that for the receive buffers);
 *   5. ep_peer_dispatch: rows, scales, local ids and weights into the owners;
 *   6. a barrier across the ranks (e.g. a one-element all-reduce on the stream),
 *      then each rank computes its experts into its expert-output buffer;
 *   7. a barrier, then ep_peer_combine on every rank.
 * Tables of peer pointers are device arrays of W device addresses (rank order),
 * each 16-byte aligned; this rank's own entry is its local buffer.  All ranks'
 * buffers have `capacity` rows.  A partition that would receive more than
 * `capacity` rows receives none: its rows are dropped and EP_DEV_CAPACITY is set
 * on every sender (ep_peer_plan), and its rows are skipped by ep_peer_combine.
 * Nothing here waits on another rank inside a kernel; the ordering comes from the
 * caller's collectives on the same stream. */

/* Bytes of a CUDA IPC memory handle (cudaIpcMemHandle_t). */
#define EP_IPC_HANDLE_BYTES 64

/* Allocate `bytes` of device memory that other processes can map, and its handle.
 * The one allocation the library makes: memory shared by IPC must be a whole
 * allocation of its own (a caching allocator's pool block would expose its
 * neighbours).  ptr: out, 256-byte aligned; handle: out, EP_IPC_HANDLE_BYTES. */
EP_API ep_status ep_ipc_alloc(size_t bytes, void** ptr, void* handle);
/* Free memory from ep_ipc_alloc (after every peer has closed its mapping). */
EP_API ep_status ep_ipc_free(void* ptr);
/* Map another process's ep_ipc_alloc memory into this one (peer access enabled). */
EP_API ep_status ep_ipc_open(const void* handle, void** ptr);
/* Unmap memory from ep_ipc_open. */
EP_API ep_status ep_ipc_close(void* ptr);

/* Step 3.  counts: device int32 [W, E], row s = rank s's num_tokens_per_expert;
 * expert_offset: device int32 [E+1] of this rank's layout.  Writes (device):
 *   dst_offset[E]        row_of[t, k] + dst_offset[e] is (t, k)'s row in rank e/(E/W)
 *   recv_count[E/W]      rows this rank receives for each of its experts
 *   recv_offset[E/W + 1] their offsets in its receive buffer (last = total rows)
 * (zeros for this rank, and EP_DEV_CAPACITY, if it would exceed `capacity`).
 * 1 <= W <= 64 dividing E; 0 <= rank < W; 0 <= capacity < 2^31.  The workspace
 * carries the status word (workspace_bytes >= 256). */
EP_API ep_status ep_peer_plan(int32_t world, int32_t rank, int32_t num_experts, const int32_t* counts,
                              const int32_t* expert_offset, int64_t capacity, int32_t* dst_offset,
                              int32_t* recv_count, int32_t* recv_offset, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Receive buffers of every rank, as tables of W device pointers (device arrays). */
typedef struct ep_peer_buffers {
    void* const* recv_x;               /* [capacity, H] E4M3 or BF16 */
    float* const* recv_scales;         /* [capacity, H/128] fp32 row-major; NULL for BF16 */
    int32_t* const* recv_topk_idx;     /* [capacity] local expert id */
    float* const* recv_topk_weights;   /* [capacity] */
    int64_t capacity;                  /* rows of each rank's arrays, < 2^31 */
} ep_peer_buffers;

/* Step 5: ep_dispatch's payload, scales and metadata for every valid (t, k),
 * written to row row_of[t, k] + dst_offset[e] of the owner's buffers (peers).
 * handle: this rank's layout from ep_get_dispatch_layout with W partitions
 * (row_of is read); quant as for ep_dispatch except EP_QUANT_SCALES_MN_MAJOR
 * (EP_ERR_INVALID_ARG).  The workspace needs only its 256-byte header (the
 * ticket counter and status word) and must not be used by another call at the
 * same time. */
EP_API ep_status ep_peer_dispatch(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                  int32_t num_experts, int32_t world, int32_t quant, const void* x,
                                  const int64_t* topk_idx, const float* topk_weights,
                                  const ep_layout* handle, const int32_t* dst_offset,
                                  const ep_peer_buffers* peers, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Step 7: ep_combine with the rows read from the owners' expert outputs:
 *   acc = +0.0f; for k = 0..K-1 with row_of[t, k] >= 0:
 *       e = topk_idx[t, k]; row = row_of[t, k] + dst_offset[e];
 *       acc = fmaf(topk_weights[t, k], float(expert_out[e / (E/W)][row, i]), acc)
 *   y[t, i] = bf16_round_to_nearest_even(acc)
 * expert_out: device table of W pointers to BF16 [capacity, H]; a row outside
 * [0, capacity) is skipped and sets EP_DEV_INDEX_RANGE.  y: BF16 [T, H]. */
EP_API ep_status ep_peer_combine(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                 int32_t num_experts, int32_t world, const void* const* expert_out,
                                 int64_t capacity, const ep_layout* handle, const int64_t* topk_idx,
                                 const int32_t* dst_offset, const float* topk_weights, void* y,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* ---- deduplicated rows across GPUs -------------------------------------------
 * DeepEP's normal kernels send a token once to each rank that holds any of its
 * experts ("deepseek.csdn.net/67bd3eb22e30c863900615cc", "使用示例": recv_topk_idx /
 * recv_topk_weights list each received token's local experts; "DeepSeek 开源周第二弹：
 * DeepEP", "DeepEP 的常规内核和低延迟内核": top-4 groups of top-8 experts), which under
 * group-limited routing roughly halves the rows that cross NVLink.  The peer form of
 * ep_dispatch_dedup / ep_combine_dedup, with W = number of ranks = partitions:
 *   1. ep_get_dispatch_layout_dedup (partition-sized handle);
 *   2. the caller gathers every rank's handle.num_tokens_per_expert[W] (rows per
 *      rank) into counts[W, W];
 *   3. ep_peer_plan(world = W, num_experts = W, counts, handle.expert_offset, ...):
 *      dst_offset[W], this rank's recv_count[1] and recv_offset[2];
 *   4. as above (the buffers this step overwrites are free);
 *   5. ep_peer_dispatch_dedup; 6. barrier, each rank computes its partition outputs
 *      (one BF16 row per received row: the weighted sum over its listed experts);
 *   7. barrier, ep_peer_combine_dedup.
 * Rank q receives its rows source rank first, then token ascending: partition q's
 * rows of the one-GPU ep_dispatch_dedup of all ranks' tokens concatenated in rank
 * order.  recv_topk_idx / recv_topk_weights tables point to [capacity, K] arrays. */

/* The deduplicated layout of ep_dispatch_dedup on its own (partition-sized handle:
 * num_tokens_per_expert[P] = rows per partition, expert_offset[P+1], row_of[T, P],
 * src_of[T*min(P, K)] = token of each row).  1 <= P <= 32. */
EP_API ep_status ep_get_dispatch_layout_dedup(int64_t num_tokens, int32_t num_topk,
                                              int32_t num_experts, int32_t num_partitions,
                                              const int64_t* topk_idx, const ep_layout* layout,
                                              void* workspace, size_t workspace_bytes,
                                              void* stream);

/* Step 5: ep_dispatch_dedup's rows (payload, scales, [K] local-id and weight lists)
 * written to row row_of[t, q] + dst_offset[q] of rank q's buffers.  handle: from
 * ep_get_dispatch_layout_dedup with W partitions; quant as for ep_peer_dispatch.
 * 1 <= W <= 32.  The workspace needs only its 256-byte header. */
EP_API ep_status ep_peer_dispatch_dedup(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                        int32_t num_experts, int32_t world, int32_t quant,
                                        const void* x, const int64_t* topk_idx,
                                        const float* topk_weights, const ep_layout* handle,
                                        const int32_t* dst_offset, const ep_peer_buffers* peers,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* Step 7: y[t, i] = bf16_rne(sum over q = 0..W-1 with row_of[t, q] >= 0, in q order, of
 * float(partition_out[q][row_of[t, q] + dst_offset[q], i])) (fp32 adds from +0.0f).
 * partition_out: device table of W pointers to BF16 [capacity, H]; a row outside
 * [0, capacity) is skipped and sets EP_DEV_INDEX_RANGE. */
EP_API ep_status ep_peer_combine_dedup(int64_t num_tokens, int64_t hidden, int32_t world,
                                       const void* const* partition_out, int64_t capacity,
                                       const ep_layout* handle, const int32_t* dst_offset,
                                       void* y, void* workspace, size_t workspace_bytes,
                                       void* stream);

/* ---- low-latency rows across GPUs ---------------------------------------------
 * deepseek.csdn.net/67bd3eb22e30c863900615cc, "推理解码阶段的应用":
 * low_latency_dispatch(hidden_states, topk_idx, num_max_tokens, num_experts) with a
 * buffer of num_max_tokens rows per expert; "DeepSeek 开源周第二弹：DeepEP",
 * "DeepEP 的常规内核和低延迟内核": low-latency kernels for decode.  The peer form,
 * in the layout of DeepEP's low-latency receive buffer: rank q holds, for each of
 * its Epp = E/W experts, W * cap rows, source rank s owning rows [s*cap, (s+1)*cap).
 * Source rank `rank` writes slot j of expert e (the slot ep_low_latency_dispatch
 * would use) to row ((e % Epp) * W + rank) * cap + j of rank e/Epp's buffer, and
 * its row count of e to entry (e % Epp) * W + rank of that rank's count table, so
 * nothing is exchanged before the dispatch.  Steps: ep_peer_low_latency_dispatch
 * on every rank; barrier; each rank computes its experts over the first
 * count[el][s] rows of each (local expert el, source s) block; barrier;
 * ep_peer_low_latency_combine on every rank.  cap = num_max_tokens >= T on every
 * rank; the handle (local: e * cap + j) is what ep_low_latency_dispatch returns. */

/* recv_x: device table of W pointers to E4M3 [E/W, W*cap, H]; recv_scales: to fp32
 * [E/W, W*cap, H/128]; recv_expert_count: to int32 [E/W, W].  Unused rows are not
 * written.  Errors as for ep_low_latency_dispatch; 0 <= rank < W, W divides E. */
EP_API ep_status ep_peer_low_latency_dispatch(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                              int32_t num_experts, int32_t world, int32_t rank,
                                              int32_t num_max_tokens, const void* x,
                                              const int64_t* topk_idx, void* const* recv_x,
                                              float* const* recv_scales,
                                              int32_t* const* recv_expert_count,
                                              const ep_ll_handle* handle, void* workspace,
                                              size_t workspace_bytes, void* stream);

/* ep_low_latency_combine with slot row e * cap + j of (t, k) read from row
 * ((e % Epp) * W + rank) * cap + j of expert_out[e / Epp] (device table of W
 * pointers to BF16 [E/W, W*cap, H]).  topk_idx: the ids the dispatch used. */
EP_API ep_status ep_peer_low_latency_combine(int64_t num_tokens, int64_t hidden, int32_t num_topk,
                                             int32_t num_experts, int32_t world, int32_t rank,
                                             int32_t num_max_tokens, const void* const* expert_out,
                                             const int64_t* topk_idx, const ep_ll_handle* handle,
                                             const float* topk_weights, void* y, void* workspace,
                                             size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_H */
