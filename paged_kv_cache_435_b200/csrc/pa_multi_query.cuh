// Internal interface between the C ABI and the multi-query kernel.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace pa {

struct MultiQueryParams {
    float* out;                     // fp32 [T][Hq][D], T = query_start_loc[B]
    const uint16_t* q;              // bf16 [T][Hq][D]
    const uint16_t* k_cache;        // bf16 [NB][bs][Hkv][D]
    const uint16_t* v_cache;
    const int32_t* block_tables;    // int32 [B][max_blocks_per_seq]
    const int32_t* context_lens;    // int32 [B]
    const int32_t* query_start_loc; // int32 [B+1]
    int* error_flags;               // nullable
    int num_seqs;
    int max_blocks_per_seq;
    int max_context_len;
    int max_query_len;
    int num_heads;
    int num_kv_heads;
    int num_blocks;
    int group;                      // num_heads / num_kv_heads
    float scale_log2;               // scale * log2(e)
};

float mq_log2e_scale(float scale);

// Row tiles (grid.y) for this shape.
int multi_query_row_tiles(int max_query_len, int group);

cudaError_t launch_paged_multi_query(const MultiQueryParams& p, int head_size,
                                     int block_size, cudaStream_t stream);

// tcgen05 kernel for 128-row tiles (pa_multi_query_tc.cu): head_size 128 and
// at least 128 (query token, head) rows per sequence.
bool multi_query_tc_eligible(int head_size, int max_query_len, int group);
cudaError_t launch_paged_multi_query_tc(const MultiQueryParams& p,
                                        int block_size, cudaStream_t stream);

}  // namespace pa
