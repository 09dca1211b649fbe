// Internal interface between the C ABI (pa_api.cu) and the decode kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "pa_cascade.cuh"

namespace pa {

struct DecodeParams {
    float* out;                  // fp32 [B][Hq][D]
    const uint16_t* q;           // bf16 [B][Hq][D]
    const uint16_t* k_cache;     // bf16 [NB][bs][Hkv][D]
    const uint16_t* v_cache;
    const int32_t* block_tables; // int32 [B][max_blocks_per_seq]
    const int32_t* context_lens; // int32 [B]
    float* tmp_o;                // fp32 [B][Hq][max_partitions][D]
    float* tmp_m;                // fp32 [B][Hq][max_partitions] (log2 domain)
    float* tmp_l;                // fp32 [B][Hq][max_partitions]
    // Persistent split grid: every warp streams its own range of chunks
    // (a "range worker"); the piece a worker starts in the middle of a
    // partition goes to the worker's straddle row.
    float* st_o;                 // fp32 [Hq][max_range_workers][D]
    float* st_m;                 // fp32 [Hq][max_range_workers]
    float* st_l;                 // fp32 [Hq][max_range_workers]
    int32_t* chunk_prefix;       // int32 [B+1]: 16-token chunks before each
                                 // sequence (written by the partition kernel)
    int32_t* worker_bounds;      // int32 [max_range_workers+1]: first chunk
                                 // position of each worker's range (likewise)
    // Merge of the range workers' pieces, in slices of kMergeRows candidate
    // rows: per (sequence, query head) an arrival counter that the partition
    // kernel zeroes, and each slice's (max, sum, normalised O).
    int32_t* merge_count;        // int32 [B][Hq]
    float* sub_o;                // fp32 [B][Hq][max_slices][D]
    float* sub_m;                // fp32 [B][Hq][max_slices]
    float* sub_l;                // fp32 [B][Hq][max_slices]
    int max_slices;
    int* error_flags;            // nullable
    int num_seqs;
    int max_blocks_per_seq;
    int max_context_len;
    int num_heads;
    int num_kv_heads;
    int num_blocks;
    int group;                   // num_heads / num_kv_heads (1..8)
    int partition_size;          // tokens, multiple of block_size
    int max_partitions;          // ceil(max_context_len / partition_size)
    float scale_log2;            // scale * log2(e)
    int block_size;
    int max_range_workers;       // rows of the straddle region per query head
    int range_workers;           // split on the persistent grid: range workers
                                 // (warps) per kv head; 0 otherwise
    // Shared-prefix call: the members of valid groups with a prefix are
    // answered by the group pass and have no items here; both passes
    // classify a sequence with the same functions (pa_cascade.cuh).
    bool has_groups;
    CascadeGroups groups;
    // Ints the partition kernel zeroes before anything else reads them (the
    // group pass's arrival counters, which it reads only after this grid).
    int32_t* zero_ints;
    long long zero_count;
};

// scale * log2(e): logits are kept in the log2 domain (exp2f).
float log2e_scale(float scale);

// CTAs per kv head of the persistent grid on the current device (about two
// per SM over all kv heads), and the range workers (warps) they hold, which
// size the straddle region.
int decode_ctas_per_head(int num_kv_heads);
int decode_range_workers(int num_kv_heads);

// Candidate rows merged by one work item of the range merge.
constexpr int kMergeRows = 64;

// Enqueue the partition kernel (and the merge kernel when
// max_partitions > 1).  head_size in {64,128}, block_size in {16,32};
// num_blocks * block_size < 2^31.
cudaError_t launch_paged_decode(const DecodeParams& p, int head_size,
                                int block_size, cudaStream_t stream);

}  // namespace pa
