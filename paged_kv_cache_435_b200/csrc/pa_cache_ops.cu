// Cache-write and copy-on-write kernels of libpagedattn.so.
//
//  reshape_and_cache: the new token's K/V rows go to slot s of the paged pool
//  (block s / block_size, offset s % block_size); the slot comes from the
//  block manager's on-demand allocation ("vLLM: Anatomy and Mechanisms of
//  High-Throughput LLM Inference", "Block-Level Management").
//
//  copy_blocks: whole-block copies for copy-on-write when blocks shared by
//  parallel samples or beams diverge (same page, "Memory Sharing via
//  Copy-on-Write (CoW)").
//
// Both are pure data movement: 16-byte vector loads/stores, one thread per
// 16 bytes, grids sized in multiples of the SM count.
#include <cstdint>

#include "pa_cache_ops.cuh"
#include "pa_common.cuh"

namespace pa {
namespace {

// One thread per (token, kv head, 16-byte chunk of head_size).
template <bool kVec>
__global__ void __launch_bounds__(256)
reshape_and_cache_kernel(const uint16_t* __restrict__ key,
                         const uint16_t* __restrict__ value,
                         int64_t key_stride, int64_t value_stride,
                         uint16_t* __restrict__ k_cache,
                         uint16_t* __restrict__ v_cache,
                         const int64_t* __restrict__ slot_mapping,
                         int num_tokens, int64_t num_slots, int block_size,
                         int num_kv_heads, int head_size, int* error_flags) {
    pdl_launch_dependents();  // a following decode launch may get scheduled
    const int chunk_elems = kVec ? 8 : 1;
    const int chunks = head_size / chunk_elems;
    const int64_t per_token = (int64_t)num_kv_heads * chunks;
    const int64_t total = (int64_t)num_tokens * per_token;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
         idx < total; idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = idx / per_token;
        const int64_t rem = idx - i * per_token;
        const int h = (int)(rem / chunks);
        const int c = (int)(rem - (int64_t)h * chunks);
        const int64_t slot = slot_mapping[i];
        if (slot < 0) continue;  // padding token
        if (slot >= num_slots) {
            if (h == 0 && c == 0) report(error_flags, PA_DEVERR_SLOT);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int64_t off = slot - blk * block_size;
        const int64_t dst =
            ((blk * block_size + off) * num_kv_heads + h) * (int64_t)head_size +
            (int64_t)c * chunk_elems;
        const int64_t ks = i * key_stride + (int64_t)h * head_size +
                           (int64_t)c * chunk_elems;
        const int64_t vs = i * value_stride + (int64_t)h * head_size +
                           (int64_t)c * chunk_elems;
        if (kVec) {
            *reinterpret_cast<uint4*>(k_cache + dst) =
                __ldg(reinterpret_cast<const uint4*>(key + ks));
            *reinterpret_cast<uint4*>(v_cache + dst) =
                __ldg(reinterpret_cast<const uint4*>(value + vs));
        } else {
            k_cache[dst] = key[ks];
            v_cache[dst] = value[vs];
        }
    }
}

// grid.x: pair, grid.y: layer within this launch's chunk, grid.z: 0=K, 1=V.
__global__ void __launch_bounds__(256)
copy_blocks_kernel(CopyLayerPtrs ptrs, const int64_t* __restrict__ mapping,
                   int64_t num_blocks, int64_t block_vecs, int* error_flags) {
    pdl_launch_dependents();
    const int p = blockIdx.x;
    const int layer = blockIdx.y;
    const int64_t src = mapping[2 * (int64_t)p];
    const int64_t dst = mapping[2 * (int64_t)p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0 && layer == 0 && blockIdx.z == 0)
            report(error_flags, PA_DEVERR_COPY_PAIR);
        return;
    }
    if (src == dst) return;
    uint4* base = reinterpret_cast<uint4*>(blockIdx.z == 0 ? ptrs.k[layer]
                                                           : ptrs.v[layer]);
    const uint4* from = base + src * block_vecs;
    uint4* to = base + dst * block_vecs;
    for (int64_t i = threadIdx.x; i < block_vecs; i += blockDim.x)
        to[i] = __ldg(from + i);
}

}  // namespace

cudaError_t launch_reshape_and_cache(const void* key, const void* value,
                                     int64_t key_stride, int64_t value_stride,
                                     void* k_cache, void* v_cache,
                                     const int64_t* slot_mapping,
                                     int num_tokens, int num_blocks,
                                     int block_size, int num_kv_heads,
                                     int head_size, int* error_flags,
                                     cudaStream_t stream) {
    const bool vec =
        (reinterpret_cast<uintptr_t>(key) % 16 == 0) &&
        (reinterpret_cast<uintptr_t>(value) % 16 == 0) &&
        (key_stride % 8 == 0) && (value_stride % 8 == 0) &&
        (head_size % 8 == 0) &&
        (reinterpret_cast<uintptr_t>(k_cache) % 16 == 0) &&
        (reinterpret_cast<uintptr_t>(v_cache) % 16 == 0);
    const int64_t work = (int64_t)num_tokens * num_kv_heads *
                         (vec ? head_size / 8 : head_size);
    const int threads = 256;
    int64_t blocks = (work + threads - 1) / threads;
    const int64_t cap = 8LL * device_sm_count();  // grid-stride beyond 8 CTAs per SM
    if (blocks > cap) blocks = cap;
    const int64_t num_slots = (int64_t)num_blocks * block_size;
    auto* k = static_cast<const uint16_t*>(key);
    auto* v = static_cast<const uint16_t*>(value);
    auto* kc = static_cast<uint16_t*>(k_cache);
    auto* vc = static_cast<uint16_t*>(v_cache);
    if (vec)
        reshape_and_cache_kernel<true><<<(unsigned)blocks, threads, 0, stream>>>(
            k, v, key_stride, value_stride, kc, vc, slot_mapping, num_tokens,
            num_slots, block_size, num_kv_heads, head_size, error_flags);
    else
        reshape_and_cache_kernel<false><<<(unsigned)blocks, threads, 0, stream>>>(
            k, v, key_stride, value_stride, kc, vc, slot_mapping, num_tokens,
            num_slots, block_size, num_kv_heads, head_size, error_flags);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void* const* k_caches, void* const* v_caches,
                               int num_layers, const int64_t* block_mapping,
                               int num_pairs, int num_blocks, int block_size,
                               int num_kv_heads, int head_size,
                               int* error_flags, cudaStream_t stream) {
    const int64_t block_bytes =
        (int64_t)block_size * num_kv_heads * head_size * 2;
    const int64_t block_vecs = block_bytes / 16;
    for (int l0 = 0; l0 < num_layers; l0 += kMaxCopyLayers) {
        const int nl = (num_layers - l0 < kMaxCopyLayers) ? num_layers - l0
                                                          : kMaxCopyLayers;
        CopyLayerPtrs ptrs;
        for (int i = 0; i < nl; ++i) {
            ptrs.k[i] = k_caches[l0 + i];
            ptrs.v[i] = v_caches[l0 + i];
        }
        dim3 grid((unsigned)num_pairs, (unsigned)nl, 2);
        copy_blocks_kernel<<<grid, 256, 0, stream>>>(
            ptrs, block_mapping, num_blocks, block_vecs, error_flags);
        count_launch();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace pa
