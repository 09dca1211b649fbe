// swap_blocks: whole-block moves between a GPU pool and a pinned CPU pool,
// the swapping form of preemption ("vLLM: Anatomy and Mechanisms of
// High-Throughput LLM Inference", "Preemption and Recovery": evicted KV
// blocks are moved to CPU RAM; "vLLM Internals", "The Block Manager": a
// request's blocks are swapped to CPU and resumed later).
//
// One zero-copy kernel serves both directions: either side may be HBM or
// pinned host memory, which the GPU addresses directly under unified
// addressing, so blocks cross PCIe / C2C as 16-byte coalesced accesses
// without per-block memcpy calls.  Each CTA moves one (pair, cache) block;
// every thread keeps 16 independent 16-byte loads in flight to cover the
// link latency of host reads.
#include <cuda_runtime.h>

#include <cstdint>

#include "pa_common.cuh"
#include "pa_swap.cuh"

namespace pa {
namespace {

constexpr int kSwapThreads = 256;
constexpr int kSwapUnroll = 16;

__global__ void __launch_bounds__(kSwapThreads)
swap_blocks_kernel(SwapPtrs ptrs, const int64_t* __restrict__ mapping,
                   int64_t src_num_blocks, int64_t dst_num_blocks,
                   int64_t block_vecs, int* error_flags) {
    const int p = blockIdx.x;
    const int c = blockIdx.y;
    const int64_t src = mapping[2 * (int64_t)p];
    const int64_t dst = mapping[2 * (int64_t)p + 1];
    if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
        if (threadIdx.x == 0 && c == 0) report(error_flags, PA_DEVERR_COPY_PAIR);
        return;
    }
    const uint4* from = reinterpret_cast<const uint4*>(ptrs.src[c]) + src * block_vecs;
    uint4* to = reinterpret_cast<uint4*>(ptrs.dst[c]) + dst * block_vecs;
    for (int64_t base = 0; base < block_vecs; base += kSwapThreads * kSwapUnroll) {
        uint4 r[kSwapUnroll];
#pragma unroll
        for (int u = 0; u < kSwapUnroll; ++u) {
            const int64_t i = base + u * kSwapThreads + threadIdx.x;
            if (i < block_vecs) r[u] = from[i];
        }
#pragma unroll
        for (int u = 0; u < kSwapUnroll; ++u) {
            const int64_t i = base + u * kSwapThreads + threadIdx.x;
            if (i < block_vecs) to[i] = r[u];
        }
    }
}

}  // namespace

cudaError_t launch_swap_blocks(const void* const* src_caches,
                               void* const* dst_caches, int num_caches,
                               const int64_t* block_mapping, int num_pairs,
                               int64_t block_bytes, int64_t src_num_blocks,
                               int64_t dst_num_blocks, int* error_flags,
                               cudaStream_t stream) {
    const int64_t block_vecs = block_bytes / 16;
    for (int c0 = 0; c0 < num_caches; c0 += kMaxSwapCaches) {
        const int nc = num_caches - c0 < kMaxSwapCaches ? num_caches - c0 : kMaxSwapCaches;
        SwapPtrs ptrs;
        for (int i = 0; i < nc; ++i) {
            ptrs.src[i] = src_caches[c0 + i];
            ptrs.dst[i] = dst_caches[c0 + i];
        }
        swap_blocks_kernel<<<dim3((unsigned)num_pairs, (unsigned)nc), kSwapThreads, 0,
                             stream>>>(ptrs, block_mapping, src_num_blocks,
                                       dst_num_blocks, block_vecs, error_flags);
        count_launch();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace pa
