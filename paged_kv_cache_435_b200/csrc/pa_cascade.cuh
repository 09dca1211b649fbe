// Shared-prefix groups ("vLLM: Anatomy and Mechanisms of High-Throughput LLM
// Inference", "Memory Sharing via Copy-on-Write (CoW)": parallel samples of
// one prompt share the prompt's KV blocks).
//
// Group i is the sequences group_start[i] .. group_start[i+1]-1, whose first
// prefix_lens[i] tokens live in the same physical blocks.  The group pass
// (pa_multi_row.cu) answers every member of a valid group with a prefix; the
// decode kernel answers the other sequences.  Both sides classify a sequence
// with the functions below from the same arrays, so they agree on every
// input, valid or not: an invalid group counts as ungrouped.
#pragma once

#include <cstdint>

#include "pa_common.cuh"

namespace pa {

struct CascadeGroups {
    const int32_t* group_start;  // int32 [num_groups + 1]
    const int32_t* prefix_lens;  // int32 [num_groups]
    int num_groups;
    int max_group_size;          // host bound; larger groups count as invalid
};

// Usable shared length of group i: prefix_lens[i] when the group lies in
// [0, num_seqs] in order, has at most max_group_size members and a length
// that is a non-negative multiple of block_size; otherwise 0.
__device__ __forceinline__ int cascade_group_prefix(const CascadeGroups& c, int i,
                                                    int num_seqs, int block_size,
                                                    int* flags, bool report_errors) {
    const int a = c.group_start[i];
    const int b = c.group_start[i + 1];
    const int P = c.prefix_lens[i];
    const bool ok = a >= 0 && a <= b && b <= num_seqs && b - a <= c.max_group_size &&
                    P >= 0 && P % block_size == 0;
    if (!ok) {
        if (report_errors) report(flags, PA_DEVERR_PREFIX);
        return 0;
    }
    return P;
}

// Group holding sequence s (the last i with group_start[i] <= s, if s is
// below group_start[i+1]), or -1.
__device__ __forceinline__ int cascade_group_of(const CascadeGroups& c, int s) {
    if (c.num_groups <= 0 || c.group_start[0] > s) return -1;
    int lo = 0, hi = c.num_groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (c.group_start[mid] <= s) lo = mid; else hi = mid - 1;
    }
    return s < c.group_start[lo + 1] ? lo : -1;
}

}  // namespace pa
