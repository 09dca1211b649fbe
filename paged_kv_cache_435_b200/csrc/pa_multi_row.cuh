// Internal interface of the tcgen05 kernel for up to 32 query rows per kv
// head (pa_multi_row.cu): speculative verification in the multi-query call
// and the group pass of the shared-prefix call.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "pa_cascade.cuh"

namespace pa {

struct MultiRowParams {
    // out fp32 [T][Hq][D] (multi-query mode) or [B][Hq][D] (shared-prefix
    // mode: the rows of the members of valid groups), normalised.
    float* out;
    const uint16_t* q;               // bf16 [T or B][Hq][D]
    const uint16_t* k_cache;         // bf16 [NB][bs][Hkv][D]
    const uint16_t* v_cache;
    const int32_t* block_tables;     // int32 [B][max_blocks_per_seq]
    const int32_t* context_lens;     // int32 [B]
    const int32_t* query_start_loc;  // int32 [B+1] (multi-query mode)
    CascadeGroups groups;            // shared-prefix mode
    int* error_flags;                // nullable
    int shared_prefix_mode;
    int num_seqs;
    int max_blocks_per_seq;
    int max_context_len;
    int max_query_len;
    int num_heads;
    int num_kv_heads;
    int num_blocks;
    int block_size;
    int group;                       // num_heads / num_kv_heads
    int tiles;                       // 32-row tiles per sequence or group
    int num_units;                   // sequences or groups
    float scale_log2;                // scale * log2(e)
    // Shared-prefix mode, optional (null: items are never split): a group's
    // item may be cut at 128-token chunk boundaries into pieces on several
    // CTAs.  A piece that does not cover the whole item writes its rows'
    // (reference, sum, normalised O)
    // to slot `unit` (the piece at the item's start) or num_units + j (the
    // piece CTA j of the head starts inside the item), and counts itself on
    // the item's arrival counter (zeroed by the launch before this one); the
    // last piece to arrive merges the item's pieces into the output.
    float* piece_o;                  // fp32 [slots][Hkv][32][D]
    float* piece_ml;                 // fp32 [slots][Hkv][32][2]
    int32_t* piece_count;            // int32 [num_units][Hkv]
    int piece_slots;                 // num_units + CTAs per kv head (at most)
};

// Rows handled per tile.
constexpr int kMultiRowTile = 32;

// head_size 128 only; block_size 16 or 32.
cudaError_t launch_paged_multi_row(const MultiRowParams& p, cudaStream_t stream);

// CTAs per kv head the kernel launches at most on the current device.
int multi_row_ctas_per_head(int num_kv_heads);

}  // namespace pa
