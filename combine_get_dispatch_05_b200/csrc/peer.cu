// peer.cu -- expert parallelism across GPUs: where one rank's rows go in the owner
// ranks' receive buffers.
//
// Pages: "DeepSeek 开源周第二弹：DeepEP", section "DeepEP 的常规内核和低延迟内核" (the
// normal kernels move tokens between the GPUs of a node over NVLink) and
// "deepseek-ai/DeepEP", section "典型工作流程" (dispatch to the ranks that hold the
// experts, expert computation, combine back).  With partitions = ranks, rank p
// owns experts [p * Epp, (p + 1) * Epp).  Its receive buffer is expert-major, then
// source rank ascending, then (token, k) ascending: the rows partition p would get
// from the one-GPU dispatch of all ranks' tokens concatenated in rank order.  For
// source rank s and expert e of partition p, the row of (t, k) there is
//     row_of_s[t, k] - expert_offset_s[e]                (rank of (t, k) in e on s)
//   + sum_{s' < s} count[s'][e]                          (rows of e from earlier ranks)
//   + sum_{e' in p, e' < e} sum_{s'} count[s'][e']       (earlier experts of p)
// so one per-expert offset, dst_offset[e], turns the local row into the remote
// one.  The plan kernel computes it from every rank's per-expert counts (gathered
// by the caller), with this rank's receive counts and offsets.  If a partition
// receives more rows than `capacity`, every offset of its experts is set so that
// all their rows fall outside the buffer (the dispatch and combine kernels then
// skip them) and EP_DEV_CAPACITY is raised.  The plan is a programmatic dependent
// of what precedes it and, once that is complete, lets the dispatch kernel start:
// the dispatch loads and quantises its rows while the plan runs, and only its storer
// waits for the offsets.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kPlanThreads = 256;
constexpr int32_t kNoRoom = 0x7fffffff;  // offset that puts every row past any buffer

// Shared memory (dynamic): total[E] (rows of expert e over all ranks) | before[E]
// (rows of e from ranks < rank) | base[E] (offset of e's segment in its owner's
// buffer) as int64.
__global__ void __launch_bounds__(kPlanThreads) peer_plan_kernel(PeerPlanParams p) {
    pdl_wait();               // the counts and the layout are complete and visible
    pdl_launch_dependents();  // the dispatch may start loading and quantising its rows
    extern __shared__ int64_t psm[];
    const int E = p.num_experts, W = p.world;
    const int epp = E / W;
    int64_t* total = psm;
    int64_t* before = total + E;
    int64_t* base = before + E;
    __shared__ int overflow[64];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int64_t sum = 0, pre = 0;
        for (int s = 0; s < W; ++s) {
            const int64_t c = p.counts[static_cast<int64_t>(s) * E + e];
            if (s < p.rank) pre += c;
            sum += c;
        }
        total[e] = sum;
        before[e] = pre;
    }
    __syncthreads();
    // one thread per partition: the segments of its experts, in expert order
    for (int q = threadIdx.x; q < W; q += blockDim.x) {
        int64_t run = 0;
        for (int j = 0; j < epp; ++j) {
            base[q * epp + j] = run;
            run += total[q * epp + j];
        }
        overflow[q] = run > p.capacity;
        if (q == p.rank) p.recv_offset[epp] = static_cast<int32_t>(run > p.capacity ? 0 : run);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int q = e / epp;
        const int64_t off = base[e] + before[e] - p.expert_offset[e];
        p.dst_offset[e] = overflow[q] ? kNoRoom : static_cast<int32_t>(off);
        if (q == p.rank) {
            const int j = e - q * epp;
            p.recv_count[j] = overflow[q] ? 0 : static_cast<int32_t>(total[e]);
            p.recv_offset[j] = overflow[q] ? 0 : static_cast<int32_t>(base[e]);
        }
    }
    if (threadIdx.x == 0) {
        for (int q = 0; q < W; ++q)
            if (overflow[q]) {
                raise_status(p.status, kDevCapacity);
                break;
            }
    }
}

}  // namespace

cudaError_t launch_peer_plan(const PeerPlanParams& p, cudaStream_t stream) {
    const size_t smem = sizeof(int64_t) * 3 * static_cast<size_t>(p.num_experts);
    cudaError_t err = cudaFuncSetAttribute(peer_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    // programmatic dependent of the previous kernel; it waits for it before reading
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kPlanThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, peer_plan_kernel, p);
}

}  // namespace ep
