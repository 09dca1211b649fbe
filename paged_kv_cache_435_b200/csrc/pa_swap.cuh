// Internal launcher for the swap kernel (pa_swap.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace pa {

// Caches handled by one swap launch (pointer arrays travel as a parameter).
constexpr int kMaxSwapCaches = 128;

struct SwapPtrs {
    const void* src[kMaxSwapCaches];
    void* dst[kMaxSwapCaches];
};

cudaError_t launch_swap_blocks(const void* const* src_caches,
                               void* const* dst_caches, int num_caches,
                               const int64_t* block_mapping, int num_pairs,
                               int64_t block_bytes, int64_t src_num_blocks,
                               int64_t dst_num_blocks, int* error_flags,
                               cudaStream_t stream);

}  // namespace pa
