// C ABI of libpagedattn.so: argument validation, the split-KV plan and the
// dispatch to the kernels.  Every check here runs on the host before any
// launch; a failed check enqueues nothing.
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <cstddef>
#include <cstdint>

#include "pa.h"
#include "pa_cache_ops.cuh"
#include "pa_common.cuh"
#include "pa_decode.cuh"
#include "pa_multi_query.cuh"
#include "pa_multi_row.cuh"
#include "pa_swap.cuh"

namespace pa {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int device_sm_count() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        v <= 0) {
        (void)cudaGetLastError();
        return 148;
    }
    return v;
}

namespace {

constexpr int kAutoPartition = 512;    // tokens per partition when splitting
constexpr int kMaxGridYZ = 65535;

bool aligned16(const void* p) {
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// True when the GPU can address `p` (device, pinned host or managed memory).
bool device_accessible(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeHost ||
           a.type == cudaMemoryTypeManaged;
}

int round_up(int x, int m) { return ((x + m - 1) / m) * m; }

bool decode_shape_supported(int num_heads, int num_kv_heads, int head_size,
                            int block_size) {
    const int G = num_heads / num_kv_heads;
    return (head_size == 64 || head_size == 128) &&
           (block_size == 16 || block_size == 32) && G >= 1 && G <= 8;
}

// Partition width in tokens (>= max_context_len means one partition).
// Split only when (sequence, kv head) units alone cannot fill the GPU with a
// few CTAs per SM; then 512-token partitions spread long contexts.
int plan_partition(int num_seqs, int num_kv_heads, int block_size,
                   int max_context_len, int partition_size) {
    if (partition_size > 0) return partition_size;
    const int whole = round_up(max_context_len > 0 ? max_context_len : 1,
                               block_size);
    if (max_context_len <= kAutoPartition) return whole;
    const long long units = (long long)num_seqs * num_kv_heads;
    if (units >= 4LL * device_sm_count()) return whole;
    int part = round_up(kAutoPartition, block_size);
    while ((max_context_len + part - 1) / part > kMaxGridYZ) part *= 2;
    return part;
}

int num_partitions(int max_context_len, int part) {
    const int n = (max_context_len + part - 1) / part;
    return n < 1 ? 1 : n;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Split-KV scratch, each region 256-byte aligned: the partition slots
// tmp_o [B][Hq][P][D], tmp_m, tmp_l [B][Hq][P]; the persistent grid's
// straddle rows st_o [Hq][n][D], st_m, st_l [Hq][n] (n = range workers per
// kv head); the chunk prefix [B+1] and the workers' range starts [n+1];
// the range merge's arrival counters [B][Hq] and slice partials
// sub_o [B][Hq][S][D], sub_m, sub_l [B][Hq][S].
struct SplitLayout {
    size_t o, m, l, st_o, st_m, st_l, prefix, bounds, count, sub_o, sub_m, sub_l,
        total;
    int range_workers, max_slices;
};

SplitLayout split_layout(int num_seqs, int num_heads, int num_kv_heads,
                         int head_size, int max_partitions) {
    SplitLayout L{};
    L.range_workers = decode_range_workers(num_kv_heads);
    if (max_partitions <= 1) return L;
    const size_t rows = (size_t)num_seqs * num_heads * max_partitions;
    const size_t st_rows = (size_t)num_heads * L.range_workers;
    size_t off = 0;
    L.o = off;      off = align256(off + rows * head_size * 4);
    L.m = off;      off = align256(off + rows * 4);
    L.l = off;      off = align256(off + rows * 4);
    L.st_o = off;   off = align256(off + st_rows * head_size * 4);
    L.st_m = off;   off = align256(off + st_rows * 4);
    L.st_l = off;   off = align256(off + st_rows * 4);
    L.prefix = off; off = align256(off + ((size_t)num_seqs + 1) * 4);
    L.bounds = off; off = align256(off + ((size_t)L.range_workers + 1) * 4);
    // A sequence's candidate rows: its partition slots plus the range
    // boundaries inside it.
    L.max_slices = (max_partitions + L.range_workers + kMergeRows - 1) / kMergeRows;
    const size_t sub_rows = (size_t)num_seqs * num_heads * L.max_slices;
    L.count = off;  off = align256(off + (size_t)num_seqs * num_heads * 4);
    L.sub_o = off;  off = align256(off + sub_rows * head_size * 4);
    L.sub_m = off;  off = align256(off + sub_rows * 4);
    L.sub_l = off;  off = align256(off + sub_rows * 4);
    L.total = off;
    return L;
}

size_t workspace_bytes_for(int num_seqs, int num_heads, int num_kv_heads,
                           int head_size, int max_partitions) {
    return split_layout(num_seqs, num_heads, num_kv_heads, head_size,
                        max_partitions).total;
}

// Shared-prefix call, after the split scratch: the group pass's pieces of
// split items, piece_o [S][Hkv][32][D], piece_ml [S][Hkv][32][2] (S = groups
// + CTAs per kv head, groups bounded by the sequences), and the items'
// arrival counters [groups][Hkv].
struct PieceLayout {
    size_t o, ml, count, total;
    int slots;
};

PieceLayout piece_layout(size_t base, int num_seqs, int num_kv_heads, int head_size) {
    PieceLayout L{};
    L.slots = num_seqs + multi_row_ctas_per_head(num_kv_heads);
    const size_t rows = (size_t)L.slots * num_kv_heads * kMultiRowTile;
    size_t off = align256(base);
    L.o = off;     off = align256(off + rows * head_size * 4);
    L.ml = off;    off = align256(off + rows * 2 * 4);
    L.count = off; off = align256(off + (size_t)num_seqs * num_kv_heads * 4);
    L.total = off;
    return L;
}

// Point the decode parameters at the split scratch inside `ws`.
void assign_split(DecodeParams& p, unsigned char* ws, const SplitLayout& L) {
    p.max_range_workers = L.range_workers;
    if (L.total == 0) return;
    p.tmp_o = reinterpret_cast<float*>(ws + L.o);
    p.tmp_m = reinterpret_cast<float*>(ws + L.m);
    p.tmp_l = reinterpret_cast<float*>(ws + L.l);
    p.st_o = reinterpret_cast<float*>(ws + L.st_o);
    p.st_m = reinterpret_cast<float*>(ws + L.st_m);
    p.st_l = reinterpret_cast<float*>(ws + L.st_l);
    p.chunk_prefix = reinterpret_cast<int32_t*>(ws + L.prefix);
    p.worker_bounds = reinterpret_cast<int32_t*>(ws + L.bounds);
    p.merge_count = reinterpret_cast<int32_t*>(ws + L.count);
    p.sub_o = reinterpret_cast<float*>(ws + L.sub_o);
    p.sub_m = reinterpret_cast<float*>(ws + L.sub_m);
    p.sub_l = reinterpret_cast<float*>(ws + L.sub_l);
    p.max_slices = L.max_slices;
}

}  // namespace
}  // namespace pa

extern "C" {

const char* pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_NO_BLOCKS: return "PA_ERR_NO_BLOCKS";
        default: return "PA_UNKNOWN_STATUS";
    }
}

int pa_version(void) { return (1 << 16) | 0; }

uint64_t pa_launch_count(void) {
    return pa::g_launches.load(std::memory_order_relaxed);
}

int pa_reshape_and_cache(const void* key, const void* value,
                         int64_t key_token_stride, int64_t value_token_stride,
                         void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens,
                         int num_blocks, int block_size, int num_kv_heads,
                         int head_size, int* error_flags, pa_stream_t stream) {
    if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 ||
        num_kv_heads <= 0 || head_size <= 0)
        return PA_ERR_INVALID_ARG;
    const int64_t row = (int64_t)num_kv_heads * head_size;
    if (key_token_stride < row || value_token_stride < row)
        return PA_ERR_INVALID_ARG;
    if (!k_cache || !v_cache) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !slot_mapping) return PA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(key) | reinterpret_cast<uintptr_t>(value) |
         reinterpret_cast<uintptr_t>(k_cache) |
         reinterpret_cast<uintptr_t>(v_cache)) & 1u)
        return PA_ERR_INVALID_ARG;  // bf16 needs 2-byte alignment
    if ((reinterpret_cast<uintptr_t>(slot_mapping) & 7u) != 0)
        return PA_ERR_INVALID_ARG;
    cudaError_t e = pa::launch_reshape_and_cache(
        key, value, key_token_stride, value_token_stride, k_cache, v_cache,
        slot_mapping, num_tokens, num_blocks, block_size, num_kv_heads,
        head_size, error_flags, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                             int head_size, int block_size,
                             int max_context_len, int partition_size) {
    (void)num_heads;
    (void)head_size;
    if (num_seqs < 0 || num_kv_heads <= 0 || block_size <= 0 ||
        max_context_len < 0 || partition_size < 0)
        return PA_ERR_INVALID_ARG;
    if (partition_size > 0 && partition_size % block_size != 0)
        return PA_ERR_INVALID_ARG;
    return pa::plan_partition(num_seqs, num_kv_heads, block_size,
                              max_context_len, partition_size);
}

size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                int head_size, int block_size,
                                int max_context_len, int partition_size) {
    const int part = pa_decode_partition_size(num_seqs, num_heads, num_kv_heads,
                                              head_size, block_size,
                                              max_context_len, partition_size);
    if (part <= 0 || num_heads <= 0 || head_size <= 0) return 0;
    return pa::workspace_bytes_for(num_seqs, num_heads, num_kv_heads, head_size,
                                   pa::num_partitions(max_context_len, part));
}

int pa_decode_attention(float* out, const void* q, const void* k_cache,
                        const void* v_cache, const int32_t* block_tables,
                        int max_blocks_per_seq, const int32_t* context_lens,
                        int max_context_len, int num_seqs, int num_heads,
                        int num_kv_heads, int head_size, int block_size,
                        int num_blocks, float scale, int partition_size,
                        void* workspace, size_t workspace_bytes,
                        int* error_flags, pa_stream_t stream) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        head_size <= 0 || block_size <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0 || partition_size < 0)
        return PA_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size)
        return PA_ERR_INVALID_ARG;
    if (partition_size > 0 && partition_size % block_size != 0)
        return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (!pa::decode_shape_supported(num_heads, num_kv_heads, head_size,
                                       block_size))
        return PA_ERR_UNSUPPORTED;
    if ((long long)num_blocks * block_size > 0x7fffffffLL)
        return PA_ERR_UNSUPPORTED;  // token slots are 32-bit TMA coordinates
    if (num_seqs == 0) return PA_OK;
    if (num_seqs > pa::kMaxGridYZ) return PA_ERR_UNSUPPORTED;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!pa::aligned16(out) || !pa::aligned16(q) || !pa::aligned16(k_cache) ||
        !pa::aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u))
        return PA_ERR_INVALID_ARG;

    const int part = pa::plan_partition(num_seqs, num_kv_heads, block_size,
                                        max_context_len, partition_size);
    const int np = pa::num_partitions(max_context_len, part);
    if (np > pa::kMaxGridYZ) return PA_ERR_INVALID_ARG;
    const pa::SplitLayout lay =
        pa::split_layout(num_seqs, num_heads, num_kv_heads, head_size, np);
    const size_t need = lay.total;
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return PA_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
            return PA_ERR_INVALID_ARG;
    }

    pa::DecodeParams p{};
    p.out = out;
    p.q = static_cast<const uint16_t*>(q);
    p.k_cache = static_cast<const uint16_t*>(k_cache);
    p.v_cache = static_cast<const uint16_t*>(v_cache);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    pa::assign_split(p, static_cast<unsigned char*>(workspace), lay);
    p.error_flags = error_flags;
    p.num_seqs = num_seqs;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.max_context_len = max_context_len;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.group = num_heads / num_kv_heads;
    p.partition_size = part;
    p.max_partitions = np;
    p.scale_log2 = pa::log2e_scale(scale);
    p.block_size = block_size;
    cudaError_t e = pa::launch_paged_decode(
        p, head_size, block_size, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_multi_query_attention(float* out, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* block_tables,
                             int max_blocks_per_seq,
                             const int32_t* context_lens, int max_context_len,
                             const int32_t* query_start_loc, int max_query_len,
                             int num_seqs, int num_heads, int num_kv_heads,
                             int head_size, int block_size, int num_blocks,
                             float scale, int* error_flags,
                             pa_stream_t stream) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        head_size <= 0 || block_size <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0 || max_query_len < 0)
        return PA_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size)
        return PA_ERR_INVALID_ARG;
    if (max_query_len > max_context_len) return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    const int G = num_heads / num_kv_heads;
    if (!((head_size == 64 || head_size == 128) &&
          (block_size == 16 || block_size == 32) && G >= 1 && G <= 64))
        return PA_ERR_UNSUPPORTED;
    if ((long long)num_blocks * block_size > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0 || max_query_len == 0) return PA_OK;
    if (num_seqs > pa::kMaxGridYZ) return PA_ERR_UNSUPPORTED;
    if ((long long)max_query_len * G > 16LL * 4 * pa::kMaxGridYZ)
        return PA_ERR_UNSUPPORTED;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens ||
        !query_start_loc)
        return PA_ERR_INVALID_ARG;
    if (!pa::aligned16(out) || !pa::aligned16(q) || !pa::aligned16(k_cache) ||
        !pa::aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u) ||
        (reinterpret_cast<uintptr_t>(query_start_loc) & 3u))
        return PA_ERR_INVALID_ARG;
    pa::MultiQueryParams p{};
    p.out = out;
    p.q = static_cast<const uint16_t*>(q);
    p.k_cache = static_cast<const uint16_t*>(k_cache);
    p.v_cache = static_cast<const uint16_t*>(v_cache);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start_loc = query_start_loc;
    p.error_flags = error_flags;
    p.num_seqs = num_seqs;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.max_context_len = max_context_len;
    p.max_query_len = max_query_len;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.group = G;
    p.scale_log2 = pa::mq_log2e_scale(scale);
    // Kernel choice (head_size 128): the 128-row tcgen05 kernel for prefill
    // chunks (>= 128 rows per sequence), the 32-row tcgen05 kernel (tokens as
    // the MMA's M) below that; head_size 64 runs on the mma.sync kernel.
    // PA_MULTI_QUERY_KERNEL=mma|tc|rows overrides the choice (tests,
    // benchmarks).
    enum { kMma, kTc, kRows } kind = kMma;
    if (pa::multi_query_tc_eligible(head_size, max_query_len, G)) kind = kTc;
    else if (head_size == 128) kind = kRows;
    if (const char* force = std::getenv("PA_MULTI_QUERY_KERNEL")) {
        if (std::strcmp(force, "mma") == 0) kind = kMma;
        if (std::strcmp(force, "tc") == 0 && head_size == 128) kind = kTc;
        if (std::strcmp(force, "rows") == 0 && head_size == 128) kind = kRows;
    }
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (kind == kRows) {
        pa::MultiRowParams r{};
        r.out = out;
        r.q = p.q;
        r.k_cache = p.k_cache;
        r.v_cache = p.v_cache;
        r.block_tables = block_tables;
        r.context_lens = context_lens;
        r.query_start_loc = query_start_loc;
        r.error_flags = error_flags;
        r.shared_prefix_mode = 0;
        r.num_seqs = num_seqs;
        r.max_blocks_per_seq = max_blocks_per_seq;
        r.max_context_len = max_context_len;
        r.max_query_len = max_query_len;
        r.num_heads = num_heads;
        r.num_kv_heads = num_kv_heads;
        r.num_blocks = num_blocks;
        r.block_size = block_size;
        r.group = G;
        r.tiles = (int)(((long long)max_query_len * G + pa::kMultiRowTile - 1) /
                        pa::kMultiRowTile);
        r.num_units = num_seqs;
        r.scale_log2 = p.scale_log2;
        if ((long long)r.num_units * r.tiles * num_kv_heads > 0x7fffffffLL)
            return PA_ERR_UNSUPPORTED;
        e = pa::launch_paged_multi_row(r, st);
    } else if (kind == kTc) {
        e = pa::launch_paged_multi_query_tc(p, block_size, st);
    } else {
        e = pa::launch_paged_multi_query(p, head_size, block_size, st);
    }
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

size_t pa_shared_prefix_workspace_size(int num_seqs, int num_heads,
                                       int num_kv_heads, int head_size,
                                       int block_size, int max_context_len,
                                       int partition_size) {
    const int part = pa_decode_partition_size(num_seqs, num_heads, num_kv_heads,
                                              head_size, block_size,
                                              max_context_len, partition_size);
    if (part <= 0 || num_heads <= 0 || head_size <= 0) return 0;
    const size_t split = pa::workspace_bytes_for(num_seqs, num_heads, num_kv_heads, head_size,
                                                 pa::num_partitions(max_context_len, part));
    return pa::piece_layout(split, num_seqs, num_kv_heads, head_size).total;
}

int pa_decode_attention_shared_prefix(
    float* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int max_context_len,
    const int32_t* group_start, const int32_t* prefix_lens, int num_groups,
    int max_group_size, int num_seqs, int num_heads, int num_kv_heads,
    int head_size, int block_size, int num_blocks, float scale,
    int partition_size, void* workspace, size_t workspace_bytes,
    int* error_flags, pa_stream_t stream) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        head_size <= 0 || block_size <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0 || partition_size < 0 ||
        num_groups < 0)
        return PA_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size)
        return PA_ERR_INVALID_ARG;
    if (partition_size > 0 && partition_size % block_size != 0)
        return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (num_groups > 0 && (max_group_size < 1 || !group_start || !prefix_lens ||
                           (reinterpret_cast<uintptr_t>(group_start) & 3u) ||
                           (reinterpret_cast<uintptr_t>(prefix_lens) & 3u)))
        return PA_ERR_INVALID_ARG;
    if (head_size != 128 ||
        !pa::decode_shape_supported(num_heads, num_kv_heads, head_size, block_size))
        return PA_ERR_UNSUPPORTED;
    if ((long long)num_blocks * block_size > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;
    if (num_seqs > pa::kMaxGridYZ) return PA_ERR_UNSUPPORTED;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!pa::aligned16(out) || !pa::aligned16(q) || !pa::aligned16(k_cache) ||
        !pa::aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u))
        return PA_ERR_INVALID_ARG;

    const int part = pa::plan_partition(num_seqs, num_kv_heads, block_size,
                                        max_context_len, partition_size);
    const int np = pa::num_partitions(max_context_len, part);
    if (np > pa::kMaxGridYZ) return PA_ERR_INVALID_ARG;
    const pa::SplitLayout lay =
        pa::split_layout(num_seqs, num_heads, num_kv_heads, head_size, np);
    const pa::PieceLayout plan = pa::piece_layout(lay.total, num_seqs, num_kv_heads, head_size);
    if (!workspace || workspace_bytes < plan.total) return PA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PA_ERR_INVALID_ARG;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const int G = num_heads / num_kv_heads;
    // A group cannot hold more than num_seqs sequences: the bound changes
    // no group's validity and keeps the grid small.
    const int mgs = max_group_size < num_seqs ? max_group_size : num_seqs;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    pa::CascadeGroups groups{group_start, prefix_lens, num_groups, mgs};
    pa::MultiRowParams r{};
    if (num_groups > 0) {
        const int per_tile = pa::kMultiRowTile / G;
        r.out = out;
        r.q = static_cast<const uint16_t*>(q);
        r.k_cache = static_cast<const uint16_t*>(k_cache);
        r.v_cache = static_cast<const uint16_t*>(v_cache);
        r.block_tables = block_tables;
        r.context_lens = context_lens;
        r.groups = groups;
        r.error_flags = error_flags;
        r.shared_prefix_mode = 1;
        r.num_seqs = num_seqs;
        r.max_blocks_per_seq = max_blocks_per_seq;
        r.max_context_len = max_context_len;
        r.num_heads = num_heads;
        r.num_kv_heads = num_kv_heads;
        r.num_blocks = num_blocks;
        r.block_size = block_size;
        r.group = G;
        r.tiles = (mgs + per_tile - 1) / per_tile;
        r.num_units = num_groups;
        r.scale_log2 = pa::log2e_scale(scale);
        if ((long long)num_groups * r.tiles * num_kv_heads > 0x7fffffffLL)
            return PA_ERR_UNSUPPORTED;
        if (num_groups <= num_seqs) {  // the piece region holds this many units
            r.piece_o = reinterpret_cast<float*>(ws + plan.o);
            r.piece_ml = reinterpret_cast<float*>(ws + plan.ml);
            r.piece_count = reinterpret_cast<int32_t*>(ws + plan.count);
            r.piece_slots = plan.slots;
        }
    }

    pa::DecodeParams p{};
    p.out = out;
    p.q = static_cast<const uint16_t*>(q);
    p.k_cache = static_cast<const uint16_t*>(k_cache);
    p.v_cache = static_cast<const uint16_t*>(v_cache);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    pa::assign_split(p, ws, lay);
    p.error_flags = error_flags;
    p.num_seqs = num_seqs;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.max_context_len = max_context_len;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.group = G;
    p.partition_size = part;
    p.max_partitions = np;
    p.scale_log2 = pa::log2e_scale(scale);
    p.block_size = block_size;
    p.has_groups = num_groups > 0;
    p.groups = groups;
    if (r.piece_count != nullptr) {
        p.zero_ints = r.piece_count;
        p.zero_count = (long long)num_groups * num_kv_heads;
    }
    // The per-sequence pass first: it attends the sequences outside every
    // group and has little to do when every sequence is grouped; the group
    // pass, launched behind it, writes the other outputs.
    if (pa::launch_paged_decode(p, head_size, block_size, st) != cudaSuccess)
        return PA_ERR_CUDA;
    if (num_groups > 0 && pa::launch_paged_multi_row(r, st) != cudaSuccess)
        return PA_ERR_CUDA;
    return PA_OK;
}

int pa_swap_blocks(const void* const* src_caches, void* const* dst_caches,
                   int num_caches, const int64_t* block_mapping, int num_pairs,
                   int64_t block_bytes, int64_t src_num_blocks,
                   int64_t dst_num_blocks, int* error_flags,
                   pa_stream_t stream) {
    if (num_caches <= 0 || num_pairs < 0 || block_bytes <= 0 ||
        block_bytes % 16 != 0 || src_num_blocks <= 0 || dst_num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (!src_caches || !dst_caches) return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!block_mapping || (reinterpret_cast<uintptr_t>(block_mapping) & 7u) ||
        !pa::device_accessible(block_mapping))
        return PA_ERR_INVALID_ARG;
    for (int c = 0; c < num_caches; ++c) {
        if (!src_caches[c] || !dst_caches[c]) return PA_ERR_INVALID_ARG;
        if (!pa::aligned16(src_caches[c]) || !pa::aligned16(dst_caches[c]))
            return PA_ERR_INVALID_ARG;
        if (!pa::device_accessible(src_caches[c]) ||
            !pa::device_accessible(dst_caches[c]))
            return PA_ERR_INVALID_ARG;
    }
    cudaError_t e = pa::launch_swap_blocks(
        src_caches, dst_caches, num_caches, block_mapping, num_pairs,
        block_bytes, src_num_blocks, dst_num_blocks, error_flags,
        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_copy_blocks(void* const* k_caches, void* const* v_caches,
                   int num_layers, const int64_t* block_mapping, int num_pairs,
                   int num_blocks, int block_size, int num_kv_heads,
                   int head_size, int* error_flags, pa_stream_t stream) {
    if (num_layers <= 0 || num_pairs < 0 || num_blocks <= 0 ||
        block_size <= 0 || num_kv_heads <= 0 || head_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (!k_caches || !v_caches) return PA_ERR_INVALID_ARG;
    for (int l = 0; l < num_layers; ++l) {
        if (!k_caches[l] || !v_caches[l]) return PA_ERR_INVALID_ARG;
        if (!pa::aligned16(k_caches[l]) || !pa::aligned16(v_caches[l]))
            return PA_ERR_INVALID_ARG;
    }
    if (((long long)block_size * num_kv_heads * head_size * 2) % 16 != 0)
        return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!block_mapping || (reinterpret_cast<uintptr_t>(block_mapping) & 7u))
        return PA_ERR_INVALID_ARG;
    cudaError_t e = pa::launch_copy_blocks(
        k_caches, v_caches, num_layers, block_mapping, num_pairs, num_blocks,
        block_size, num_kv_heads, head_size, error_flags,
        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"
