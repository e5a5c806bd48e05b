// lb.cu -- redundant experts: weight prefetch into replica slots and the gradient
// reduce over a primary and its replicas.
//
// Pages: "deepseek-ai/DeepEP" (agentlenshq.com), section "主要特性" (redundant-expert
// support through lb_prefetch_weights / lb_reduce_grads) and section "典型工作流程",
// step 5 (optionally replicate heavily loaded experts across NVLink-connected GPUs).
// On one GPU the expert slots stand for the ranks' slots; primary_of[s] names the
// slot holding slot s's authoritative copy (a primary names itself):
//   prefetch: every replica slot receives a byte copy of its primary's weight blob;
//   reduce:   the fp32 gradients of a primary and its replicas are summed in
//             ascending slot order (the first slot's value, then one add per
//             further slot) and the sum is written to every slot of the group.
// A slot whose primary_of entry is out of range or names a non-primary is skipped
// and sets the index-range status bit.
//
// Both are HBM streams: a persistent grid walks work items -- (replica slot, chunk)
// for the prefetch, (group of more than one slot, chunk) for the reduce -- and
// each thread keeps 8 (prefetch) or up to 20 (reduce) 16-byte loads in flight.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {

namespace {

constexpr int kLbThreads = 256;
constexpr int kCopyUnroll = 8;                                           // 16-byte loads in flight
constexpr int64_t kCopyChunk = int64_t(kLbThreads) * 16 * kCopyUnroll;  // bytes per work item
constexpr int kReduceBatch = 4;  // further members loaded per pass (larger groups take more passes)

__device__ __forceinline__ bool lb_valid(const int32_t* primary_of, int S, int s) {
    const int q = primary_of[s];
    return q >= 0 && q < S && primary_of[q] == q;
}

__global__ void __launch_bounds__(kLbThreads) lb_prefetch_kernel(int S, int64_t nbytes,
                                                                 const int32_t* __restrict__ primary_of,
                                                                 uint8_t* weights, uint32_t* status) {
    const int64_t nchunks = (nbytes + kCopyChunk - 1) / kCopyChunk;
    const int64_t items = static_cast<int64_t>(S) * nchunks;
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
        const int s = static_cast<int>(it / nchunks);
        const int64_t c = it - static_cast<int64_t>(s) * nchunks;
        if (!lb_valid(primary_of, S, s)) {
            if (c == 0 && threadIdx.x == 0) raise_status(status, kDevIndexRange);
            continue;
        }
        const int q = primary_of[s];
        if (q == s) continue;  // a primary keeps its weights
        const uint8_t* src = weights + static_cast<int64_t>(q) * nbytes + c * kCopyChunk;
        uint8_t* dst = weights + static_cast<int64_t>(s) * nbytes + c * kCopyChunk;
        const int64_t len = min(kCopyChunk, nbytes - c * kCopyChunk);
        uint4 v[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t off = (static_cast<int64_t>(u) * kLbThreads + threadIdx.x) * 16;
            if (off < len) v[u] = ld_stream_v4(src + off);
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t off = (static_cast<int64_t>(u) * kLbThreads + threadIdx.x) * 16;
            if (off < len) *reinterpret_cast<uint4*>(dst + off) = v[u];
        }
    }
}

// Prologue (every CTA, identically): from primary_of build the groups with more
// than one member and each group's member slots in ascending order (a stable
// counting sort of the valid slots by primary, one warp ranking 32 slots at a time).
// Work item = (group, chunk of kLbThreads * 4 float4 of the rows); groups of one
// need no work.  Shared memory (ints): po[S] | cnt[S] | off[S] | run[S] | mem[S] |
// groups[S] | ngroups.
__global__ void __launch_bounds__(kLbThreads) lb_reduce_kernel(int S, int64_t n,
                                                               const int32_t* __restrict__ primary_of,
                                                               float* grads, uint32_t* status) {
    extern __shared__ int lsm[];
    int* po = lsm;
    int* cnt = po + S;
    int* off = cnt + S;
    int* run = off + S;
    int* mem = run + S;
    int* groups = mem + S;
    int* ngroups = groups + S;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int s = tid; s < S; s += blockDim.x) {
        po[s] = primary_of[s];
        cnt[s] = 0;
        run[s] = 0;
    }
    __syncthreads();
    for (int s = tid; s < S; s += blockDim.x) {
        const int q = po[s];
        const bool ok = q >= 0 && q < S && po[q] == q;
        if (!ok) {
            po[s] = -1;  // skipped from here on
            if (blockIdx.x == 0) raise_status(status, kDevIndexRange);
        }
    }
    __syncthreads();
    for (int s = tid; s < S; s += blockDim.x)
        if (po[s] >= 0) atomicAdd(&cnt[po[s]], 1);
    __syncthreads();
    if (warp == 0) {
        // exclusive scan of the counts over primaries, and the list of groups > 1
        int carry = 0, gcarry = 0;
        for (int q0 = 0; q0 < S; q0 += 32) {
            const int q = q0 + lane;
            const int c = q < S ? cnt[q] : 0;
            int x = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (q < S) off[q] = carry + x - c;
            carry += __shfl_sync(0xffffffffu, x, 31);
            const unsigned big = __ballot_sync(0xffffffffu, c > 1);
            if (c > 1) groups[gcarry + __popc(big & ((1u << lane) - 1u))] = q;
            gcarry += __popc(big);
        }
        if (lane == 0) *ngroups = gcarry;
        // members in ascending slot order: rank among equal primaries in the batch
        for (int s0 = 0; s0 < S; s0 += 32) {
            const int s = s0 + lane;
            const int q = s < S ? po[s] : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, q);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            if (q >= 0) mem[off[q] + run[q] + rank] = s;
            __syncwarp();
            if (q >= 0 && rank == 0) run[q] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();

    const int64_t n4 = n / 4;  // float4 per row
    constexpr int kVecPerThread = 4;
    const int64_t chunk = static_cast<int64_t>(kLbThreads) * kVecPerThread;
    const int64_t nchunks = (n4 + chunk - 1) / chunk;
    const int64_t items = static_cast<int64_t>(*ngroups) * nchunks;
    float4* g = reinterpret_cast<float4*>(grads);
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
        const int gi = static_cast<int>(it / nchunks);
        const int64_t c = it - static_cast<int64_t>(gi) * nchunks;
        const int q = groups[gi];
        const int* m_list = mem + off[q];
        const int m = cnt[q];
        // all kVecPerThread vectors of the first member, then kReduceBatch members at
        // a time for all of them: up to (1 + kReduceBatch) * kVecPerThread loads in flight
        int64_t v[kVecPerThread];
        float4 acc[kVecPerThread];
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) {
            v[u] = c * chunk + static_cast<int64_t>(u) * kLbThreads + tid;
            if (v[u] < n4) acc[u] = g[static_cast<int64_t>(m_list[0]) * n4 + v[u]];
        }
        for (int j0 = 1; j0 < m; j0 += kReduceBatch) {
            float4 x[kReduceBatch][kVecPerThread];
#pragma unroll
            for (int j = 0; j < kReduceBatch; ++j)
#pragma unroll
                for (int u = 0; u < kVecPerThread; ++u)
                    if (j0 + j < m && v[u] < n4)
                        x[j][u] = g[static_cast<int64_t>(m_list[j0 + j]) * n4 + v[u]];
#pragma unroll
            for (int j = 0; j < kReduceBatch; ++j)  // ascending member order
#pragma unroll
                for (int u = 0; u < kVecPerThread; ++u)
                    if (j0 + j < m && v[u] < n4) {
                        acc[u].x = __fadd_rn(acc[u].x, x[j][u].x);
                        acc[u].y = __fadd_rn(acc[u].y, x[j][u].y);
                        acc[u].z = __fadd_rn(acc[u].z, x[j][u].z);
                        acc[u].w = __fadd_rn(acc[u].w, x[j][u].w);
                    }
        }
        for (int j = 0; j < m; ++j)
#pragma unroll
            for (int u = 0; u < kVecPerThread; ++u)
                if (v[u] < n4) g[static_cast<int64_t>(m_list[j]) * n4 + v[u]] = acc[u];
    }
}

int lb_grid(int64_t items, int num_sms) {
    const int64_t g = static_cast<int64_t>(num_sms) * 8;
    return static_cast<int>(items < g ? (items > 0 ? items : 1) : g);
}

}  // namespace

cudaError_t launch_lb_prefetch(int32_t S, int64_t nbytes, const int32_t* primary_of, void* weights,
                               uint32_t* status, cudaStream_t stream) {
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const int64_t items = static_cast<int64_t>(S) * ((nbytes + kCopyChunk - 1) / kCopyChunk);
    lb_prefetch_kernel<<<lb_grid(items, dev.num_sms), kLbThreads, 0, stream>>>(
        S, nbytes, primary_of, static_cast<uint8_t*>(weights), status);
    return cudaGetLastError();
}

cudaError_t launch_lb_reduce(int32_t S, int64_t n, const int32_t* primary_of, float* grads,
                             uint32_t* status, cudaStream_t stream) {
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    const int64_t chunk = int64_t(kLbThreads) * 4;
    // at most S / 2 groups have work; the grid covers every SM regardless
    const int64_t items = static_cast<int64_t>(S / 2 > 0 ? S / 2 : 1) * ((n / 4 + chunk - 1) / chunk);
    const size_t smem = sizeof(int) * (6 * static_cast<size_t>(S) + 1);
    err = cudaFuncSetAttribute(lb_reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    lb_reduce_kernel<<<lb_grid(items, dev.num_sms), kLbThreads, smem, stream>>>(S, n, primary_of,
                                                                              grads, status);
    return cudaGetLastError();
}

}  // namespace ep
