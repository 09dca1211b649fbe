// pa_decode_attention_static_ws: decode attention for callers that cannot
// allocate device memory.
//
// Some callers are handed only their input and output buffers and may not
// allocate anything themselves: plugin hooks inside inference runtimes,
// processes whose device memory is reserved up front by another allocator,
// or C code with no device allocator of its own.  For them this entry point
// takes its split-KV scratch from a fixed array that lives in the library's
// own device image instead of a caller-provided workspace.
//
// The array is a file-scope __device__ variable, so every GPU on which the
// library is used holds PA_STATIC_WORKSPACE_BYTES of it until the process
// exits.  Host code cannot pass the variable's name to a kernel (on the host
// it is only a stand-in for the symbol); its device address is looked up on
// every call with cudaGetSymbolAddress on the current device.  The lookup
// allocates nothing and is cheap, and it stays right when a context is torn
// down and created again (the module then reloads, possibly elsewhere).
//
// All calls share the array and it keeps whatever the last call left in it.
// The decode kernels write every scratch value before they read it within a
// call, so nothing needs clearing; calls that overlap on the GPU (for example
// on two streams at once) race on the array and must be serialised by the
// caller.
#include <cuda_runtime.h>

#include <cstddef>

#include "pa.h"

namespace {

__device__ __align__(256) unsigned char g_decode_scratch[PA_STATIC_WORKSPACE_BYTES];

// Device address of g_decode_scratch on the current device.
cudaError_t scratch_address(void** addr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    *addr = p;
    return cudaSuccess;
}

}  // namespace

extern "C" int pa_decode_attention_static_ws(
    float* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int max_context_len, int num_seqs,
    int num_heads, int num_kv_heads, int head_size, int block_size,
    int num_blocks, float scale, int partition_size, int* error_flags,
    pa_stream_t stream) {
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return PA_ERR_CUDA;
    const size_t need = pa_decode_workspace_size(
        num_seqs, num_heads, num_kv_heads, head_size, block_size,
        max_context_len, partition_size);
    if (need > (size_t)PA_STATIC_WORKSPACE_BYTES) return PA_ERR_WORKSPACE;
    return pa_decode_attention(out, q, k_cache, v_cache, block_tables,
                               max_blocks_per_seq, context_lens,
                               max_context_len, num_seqs, num_heads,
                               num_kv_heads, head_size, block_size, num_blocks,
                               scale, partition_size, scratch,
                               (size_t)PA_STATIC_WORKSPACE_BYTES, error_flags,
                               stream);
}
