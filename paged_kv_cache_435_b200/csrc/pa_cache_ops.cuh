// Internal launchers for the cache kernels (host side of pa_cache_ops.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace pa {

// Layers handled by one copy_blocks launch (pointer arrays travel as a
// kernel parameter).
constexpr int kMaxCopyLayers = 128;

struct CopyLayerPtrs {
    void* k[kMaxCopyLayers];
    void* v[kMaxCopyLayers];
};

cudaError_t launch_reshape_and_cache(const void* key, const void* value,
                                     int64_t key_stride, int64_t value_stride,
                                     void* k_cache, void* v_cache,
                                     const int64_t* slot_mapping,
                                     int num_tokens, int num_blocks,
                                     int block_size, int num_kv_heads,
                                     int head_size, int* error_flags,
                                     cudaStream_t stream);

cudaError_t launch_copy_blocks(void* const* k_caches, void* const* v_caches,
                               int num_layers, const int64_t* block_mapping,
                               int num_pairs, int num_blocks, int block_size,
                               int num_kv_heads, int head_size,
                               int* error_flags, cudaStream_t stream);

}  // namespace pa
