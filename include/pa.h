/*
 * pa.h - C ABI of libpagedattn.so: paged decode attention and its two cache
 * companions, hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * The method.  The KV cache of every sequence is kept in fixed-size,
 * non-contiguous physical blocks; a per-sequence block table maps logical
 * block i of the sequence to a physical block id, and blocks are handed out
 * on demand from a free pool ("vLLM: Anatomy and Mechanisms of High-Throughput
 * LLM Inference", section "PagedAttention: The vLLM Innovation" /
 * "Block-Level Management"; "vLLM Internals", section "The Block Manager").
 * A decode step attends with one new query token per sequence over that
 * sequence's cached context (first page, "Prefill vs. Decode Operations";
 * decode is memory-bandwidth bound there and in "The Roofline Model").
 * Sequences may share physical blocks; when a shared block diverges, only
 * that block is copied (first page, "Memory Sharing via Copy-on-Write
 * (CoW)").  One block of K and V occupies
 * 2 * block_size * num_kv_heads * head_size * 2 bytes in bf16 ("Inside vLLM:
 * Anatomy of a High-Throughput LLM Inference System", section "LLM Engine
 * constructor", KV-cache manager).
 *
 * Data layout shared by every call (all device memory, row-major):
 *   k_cache, v_cache  bf16 [num_blocks][block_size][num_kv_heads][head_size],
 *                     contiguous, base address 16-byte aligned.  Token slot
 *                     s = block_id * block_size + offset.
 *   block_tables      int32 [num_seqs][max_blocks_per_seq]; entry i of row s
 *                     is the physical block holding tokens
 *                     [i*block_size, (i+1)*block_size) of sequence s.  Entries
 *                     at or past ceil(context_lens[s] / block_size) are never
 *                     read (they may hold -1).
 *   context_lens      int32 [num_seqs]; tokens in the context of sequence s,
 *                     INCLUDING the current token (whose K/V a prior
 *                     pa_reshape_and_cache wrote).  0 means an empty context.
 *   q                 bf16 [num_seqs][num_heads][head_size], contiguous.
 *   out               fp32 [num_seqs][num_heads][head_size], contiguous.
 *
 * GQA grouping: query head h reads kv head h / (num_heads / num_kv_heads)
 * (contiguous groups; the pages name num_kv_heads but not the mapping).
 *
 * Conventions.
 *   - Ownership: the caller owns every buffer, including the workspace.  The
 *     library never allocates or frees device memory and keeps no state
 *     between calls other than a process-wide launch counter.
 *   - Asynchrony: every call only enqueues work on `stream` (0 = the legacy
 *     default stream) and returns; it never synchronises the host.
 *   - Host-side validation happens before any launch; on failure nothing is
 *     enqueued and a negative pa_status is returned.
 *   - Device-side checks: every block id, slot and context length read from
 *     device memory is bounds-checked in the kernel.  A violation never
 *     touches memory outside the caller's buffers: the access is redirected
 *     or skipped, the affected outputs are unspecified, and the matching
 *     PA_DEVERR_* bit is OR-ed into *error_flags when error_flags is non-NULL
 *     (a device int the caller zeroes and reads after the stream completes).
 *   - pa_decode_attention supports head_size in {64, 128}, block_size in
 *     {16, 32}, num_heads / num_kv_heads in 1..8 and
 *     num_blocks * block_size < 2^31; other values return PA_ERR_UNSUPPORTED.
 *     The cache ops accept any positive sizes.
 */
#ifndef PAGEDATTN_B200_PA_H
#define PAGEDATTN_B200_PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle; identical to cudaStream_t / CUstream. */
typedef struct CUstream_st* pa_stream_t;

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = -1, /* null pointer, bad size, misaligned buffer */
    PA_ERR_UNSUPPORTED = -2, /* valid but not implemented (head_size...) */
    PA_ERR_WORKSPACE = -3,   /* workspace missing or smaller than needed */
    PA_ERR_CUDA = -4,        /* the CUDA runtime reported a launch error */
    PA_ERR_NO_BLOCKS = -5    /* the block manager has too few free blocks */
} pa_status;

/* Bits OR-ed into *error_flags by the kernels. */
#define PA_DEVERR_BLOCK_ID 0x1    /* block-table entry outside [0,num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 0x2 /* context_lens[s] < 0 or > max_context_len */
#define PA_DEVERR_SLOT 0x4        /* slot_mapping entry >= num_blocks*block_size */
#define PA_DEVERR_COPY_PAIR 0x8   /* block_mapping id outside [0,num_blocks) */
#define PA_DEVERR_TIMEOUT 0x10    /* an async-copy wait exceeded its time limit */
#define PA_DEVERR_INTERNAL 0x20   /* shared memory not 1024-byte aligned (no work done) */
#define PA_DEVERR_QUERY_LEN 0x40  /* query count < 0, > context length or > max_query_len */
#define PA_DEVERR_PREFIX 0x80     /* a shared-prefix group description is invalid */

/* Human-readable name of a pa_status value (static string, never NULL). */
const char* pa_status_string(int status);

/* ABI version: (major << 16) | minor. */
int pa_version(void);

/* Number of kernels this library has launched in this process so far
 * (monotonic; lets a caller count the library's launches in a region). */
uint64_t pa_launch_count(void);

/*
 * pa_reshape_and_cache - write each new token's K and V rows into its cache
 * slot.  For token i with s = slot_mapping[i] >= 0:
 *     k_cache[s / block_size][s % block_size][h][:] = key[i][h][:]
 *     v_cache[s / block_size][s % block_size][h][:] = value[i][h][:]
 * for every kv head h.  s < 0 marks a padding token and is skipped.  This is
 * the cache write behind on-demand slot allocation ("Block-Level
 * Management"; "Allocate, reshape and bind KV cache tensors" under "LLM
 * Engine constructor" on the second page).  The copy is bit-exact.
 *
 *   key, value           bf16 [num_tokens][num_kv_heads][head_size] with a
 *                        token stride of key_token_stride / value_token_stride
 *                        ELEMENTS (>= num_kv_heads*head_size); heads and
 *                        dims are contiguous within a token.
 *   k_cache, v_cache     the pool (layout above), written in place.
 *   slot_mapping         int64 [num_tokens], device.
 *   num_tokens           >= 0 (0 enqueues nothing and returns PA_OK).
 *   error_flags          nullable device int; PA_DEVERR_SLOT on a slot
 *                        >= num_blocks*block_size (that token is skipped).
 * Two tokens mapping to the same slot is a caller error (last writer is
 * unspecified).  Returns PA_OK or a negative pa_status.
 */
int pa_reshape_and_cache(const void* key, const void* value,
                         int64_t key_token_stride, int64_t value_token_stride,
                         void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens,
                         int num_blocks, int block_size, int num_kv_heads,
                         int head_size, int* error_flags, pa_stream_t stream);

/*
 * pa_decode_partition_size - the KV partition width, in tokens, that
 * pa_decode_attention uses for these arguments (resolves partition_size = 0
 * to the library heuristic).  A result >= max_context_len means one
 * partition per sequence (no split).  Pure host function.
 */
int pa_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                             int head_size, int block_size,
                             int max_context_len, int partition_size);

/*
 * pa_decode_workspace_size - bytes of device workspace pa_decode_attention
 * needs for the same arguments (0 when no split is used).  Pure host function.
 */
size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                int head_size, int block_size,
                                int max_context_len, int partition_size);

/*
 * pa_decode_attention - paged decode attention, one query token per sequence.
 * For each sequence s with L = context_lens[s] and each query head h
 * (kv head g = h / (num_heads/num_kv_heads)):
 *     k_t = k_cache[block_tables[s][t / block_size]][t % block_size][g][:]
 *     z_t = scale * dot(q[s][h][:], k_t)              for t in [0, L)
 *     out[s][h][:] = sum_t softmax(z)_t * v_t          (fp32)
 * and out[s][h][:] = 0 when L = 0.  The gather through the block table is
 * the one the pages describe: logical block i of a sequence lives in
 * whichever physical block its table names ("vLLM: Anatomy and Mechanisms of
 * High-Throughput LLM Inference", "Block-Level Management"; "vLLM
 * Internals", "The Block Manager"), and the step streams the whole cached
 * context once, which makes it bandwidth bound (first page, "Prefill vs.
 * Decode Operations", "The Roofline Model").
 *
 * Work unit: one (sequence, KV partition) for one kv head, which reads each
 * of its blocks once for all query heads of the group.  Without a split the
 * grid has one CTA per (kv head, sequence).  When contexts are split into
 * partitions (partition_size below max_context_len), a persistent grid of
 * about two CTAs per SM walks the compact list of (sequence, partition)
 * items of each kv head (no CTA is spent past a sequence's end; above 768
 * sequences a plain grid of one CTA per (kv head, partition, sequence) with
 * early exit is used instead), and the partitions' (max, sum, normalised
 * partial output) are merged by a second kernel.
 *
 *   max_blocks_per_seq   row length of block_tables (>= 1).
 *   max_context_len      host-known upper bound of context_lens
 *                        (<= max_blocks_per_seq*block_size); sizes the split.
 *   scale                logit scale (e.g. 1/sqrt(head_size)).
 *   partition_size       0: library heuristic; otherwise the partition width
 *                        in tokens, a positive multiple of block_size.
 *   workspace            device buffer of at least
 *                        pa_decode_workspace_size(...) bytes, 256-byte
 *                        aligned (may be NULL when that size is 0).  Its
 *                        contents need no initialisation and are scratch.
 *   error_flags          nullable device int (PA_DEVERR_BLOCK_ID,
 *                        PA_DEVERR_CONTEXT_LEN, PA_DEVERR_TIMEOUT).
 * Returns PA_OK or a negative pa_status.  Run-to-run results are bitwise
 * deterministic for identical arguments.
 */
int pa_decode_attention(float* out, const void* q, const void* k_cache,
                        const void* v_cache, const int32_t* block_tables,
                        int max_blocks_per_seq, const int32_t* context_lens,
                        int max_context_len, int num_seqs, int num_heads,
                        int num_kv_heads, int head_size, int block_size,
                        int num_blocks, float scale, int partition_size,
                        void* workspace, size_t workspace_bytes,
                        int* error_flags, pa_stream_t stream);

/*
 * pa_multi_query_attention - paged attention of k new query tokens per
 * sequence, causal within the chunk: the attention of a chunked-prefill chunk
 * or of speculative-decoding verification, where all k proposed tokens are
 * checked in one pass ("vLLM: Anatomy and Mechanisms of High-Throughput LLM
 * Inference", sections "Chunked Prefill" and "Speculative Decoding"; "Inside
 * vLLM: Anatomy of a High-Throughput LLM Inference System", "Scheduler").
 *
 * Sequence s has L = context_lens[s] cached tokens, the last
 * k = query_start_loc[s+1] - query_start_loc[s] of which are its queries
 * (their K/V already written, e.g. by pa_reshape_and_cache).  Query token j
 * of s is row t = query_start_loc[s] + j of q / out; it sits at position
 * L - k + j and, for each query head h (kv head g = h / (num_heads /
 * num_kv_heads)), computes
 *     out[t][h][:] = sum_{u <= L-k+j} softmax_u(scale * q[t][h].k_u) v_u.
 * k = 1 for every sequence is decode attention.
 *
 *   q                   bf16 [T][num_heads][head_size], T = query_start_loc[num_seqs]
 *   out                 fp32 [T][num_heads][head_size]
 *   query_start_loc     int32 [num_seqs + 1], device, non-decreasing, [0] = 0
 *   max_query_len       host-known upper bound of k (<= max_context_len)
 *   other arguments     as for pa_decode_attention (no workspace: no split)
 *   error_flags         nullable; PA_DEVERR_BLOCK_ID, PA_DEVERR_CONTEXT_LEN,
 *                       PA_DEVERR_QUERY_LEN, PA_DEVERR_TIMEOUT
 * Supports head_size in {64, 128}, block_size in {16, 32},
 * num_heads / num_kv_heads in 1..64.  Returns PA_OK or a negative pa_status.
 * The kernel follows from the shape (head_size 128: a 128-row tensor-core
 * kernel when max_query_len * group >= 128, else a 32-row one; head_size
 * 64: a warp-level MMA kernel); the environment variable
 * PA_MULTI_QUERY_KERNEL = mma | tc | rows forces one of them (tests,
 * benchmarks).  Every choice computes the same function.
 */
int pa_multi_query_attention(float* out, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* block_tables,
                             int max_blocks_per_seq,
                             const int32_t* context_lens, int max_context_len,
                             const int32_t* query_start_loc, int max_query_len,
                             int num_seqs, int num_heads, int num_kv_heads,
                             int head_size, int block_size, int num_blocks,
                             float scale, int* error_flags,
                             pa_stream_t stream);

/*
 * pa_decode_attention_shared_prefix - decode attention for batches whose
 * sequences share prompt blocks, as parallel samples of one prompt or beams
 * with a common history do ("vLLM: Anatomy and Mechanisms of High-Throughput
 * LLM Inference", "Memory Sharing via Copy-on-Write (CoW)": the outputs of
 * one prompt share the prompt's KV blocks).  The result is that of
 * pa_decode_attention on the same arguments; the pages share the memory, and
 * this call also shares the reading of it.
 *
 * Group i is the sequences group_start[i] .. group_start[i+1]-1.  Their
 * block tables agree on the shared blocks: the first prefix_lens[i] /
 * block_size entries, or all entries of a member whose context is shorter;
 * the library reads them from the table of one member whose context covers
 * them.  For each (group, kv head) a group pass on the tcgen05
 * tensor cores (up to 32 query rows per pass) streams the shared blocks once
 * for all members' query rows, then each member's private tail for that
 * member's rows only: sequence s with context length L attends its first
 * min(prefix_lens[i], L) tokens through the shared blocks and the rest
 * through its own table, in one online softmax.  When there are at most 256
 * groups, each fits one pass (at most 32 / (num_heads / num_kv_heads)
 * members) and one pass alone is longer than 1.5 times an SM's even share
 * of the kv head's work, the passes are dealt to the SMs by 128-token
 * chunks: a long pass is cut into pieces on several SMs, whose partial (max,
 * sum, output) rows are merged by the piece that finishes last.  Sequences
 * outside every group, and groups whose description is invalid (reported
 * with PA_DEVERR_PREFIX), are attended by the decode kernel as by
 * pa_decode_attention.
 *
 *   group_start     int32 [num_groups + 1], device, non-decreasing, in
 *                   [0, num_seqs]; groups need not cover every sequence.
 *   prefix_lens     int32 [num_groups], device: shared tokens of each group,
 *                   a non-negative multiple of block_size (0 = no sharing).
 *   num_groups      >= 0 (0 is exactly pa_decode_attention).
 *   max_group_size  host-known upper bound of the group sizes (>= 1 when
 *                   num_groups > 0); a larger group is reported and runs
 *                   without the group pass.
 *   workspace       device buffer of at least
 *                   pa_shared_prefix_workspace_size(...) bytes, 256-byte
 *                   aligned; scratch, needs no initialisation.  It holds
 *                   the per-sequence pass's split-KV scratch, then the
 *                   group pass's pieces: (num_seqs + SMs / num_kv_heads)
 *                   x num_kv_heads x 32 rows of head_size + 2 floats, and
 *                   num_seqs x num_kv_heads arrival counters, which the
 *                   per-sequence pass clears.  The size depends on the
 *                   current device's SM count: query it on the device the
 *                   call runs on.
 *   other arguments as for pa_decode_attention.
 * The per-sequence pass runs first, then the group pass; they write
 * disjoint outputs and classify every sequence with the same rule from
 * group_start / prefix_lens, so the group pass reads nothing of the
 * per-sequence pass's but the cleared counters.
 * Supports head_size 128, block_size in {16, 32}, num_heads / num_kv_heads
 * in 1..8 (head_size 64 returns PA_ERR_UNSUPPORTED).  Returns PA_OK or a
 * negative pa_status; run-to-run results are bitwise deterministic.
 */
size_t pa_shared_prefix_workspace_size(int num_seqs, int num_heads,
                                       int num_kv_heads, int head_size,
                                       int block_size, int max_context_len,
                                       int partition_size);

int pa_decode_attention_shared_prefix(
    float* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int max_context_len,
    const int32_t* group_start, const int32_t* prefix_lens, int num_groups,
    int max_group_size, int num_seqs, int num_heads, int num_kv_heads,
    int head_size, int block_size, int num_blocks, float scale,
    int partition_size, void* workspace, size_t workspace_bytes,
    int* error_flags, pa_stream_t stream);

/*
 * pa_swap_blocks - move whole KV blocks between pools in different memories:
 * the swapping form of preemption, where evicted blocks go to CPU RAM and
 * come back when the request resumes ("vLLM: Anatomy and Mechanisms of
 * High-Throughput LLM Inference", "Preemption and Recovery"; "vLLM
 * Internals", "The Block Manager").  For each pair p and cache c:
 *     dst_caches[c][dst] = src_caches[c][src],  (src, dst) = block_mapping[p]
 * each block block_bytes bytes (2 * block_size * num_kv_heads * head_size for
 * one K or V pool of bf16), bit-exact.  One kernel serves both directions:
 * every pointer may be device memory or pinned (page-locked, registered) host
 * memory, which the GPU reads and writes directly.
 *
 *   src_caches, dst_caches  HOST arrays of num_caches pointers (e.g. the K and
 *                           V pools of every layer), 16-byte aligned;
 *                           source pools hold src_num_blocks blocks,
 *                           destination pools dst_num_blocks.
 *   block_mapping           int64 [num_pairs][2], device or pinned host.
 *   block_bytes             multiple of 16.
 *   error_flags             nullable; PA_DEVERR_COPY_PAIR on an id out of
 *                           range (that pair is skipped).
 * Pageable (unregistered) host memory is rejected with PA_ERR_INVALID_ARG.
 * No destination block may appear twice.  Returns PA_OK or a negative
 * pa_status.
 */
int pa_swap_blocks(const void* const* src_caches, void* const* dst_caches,
                   int num_caches, const int64_t* block_mapping, int num_pairs,
                   int64_t block_bytes, int64_t src_num_blocks,
                   int64_t dst_num_blocks, int* error_flags,
                   pa_stream_t stream);

/* ------------------------------------------------------------------------
 * Host-side block manager (no GPU work; not thread-safe: one owner thread).
 *
 * It keeps the free block pool (a FIFO queue: freed blocks join the back,
 * allocation takes the front), a block table per sequence, per-block
 * reference counts for sharing, optional prefix caching and a CPU pool for
 * swapping, and emits exactly the inputs the kernels above take: slot
 * mappings for pa_reshape_and_cache, block tables for the attention calls,
 * (src, dst) pairs for pa_copy_blocks and pa_swap_blocks.  Method: "vLLM:
 * Anatomy and Mechanisms of High-Throughput LLM Inference", sections
 * "Block-Level Management", "Memory Sharing via Copy-on-Write (CoW)",
 * "Preemption and Recovery", "Prefix Caching"; "Inside vLLM: Anatomy of a
 * High-Throughput LLM Inference System", KV-cache manager (free_block_queue,
 * allocate_slots); "vLLM Internals", "The Block Manager".
 * ---------------------------------------------------------------------- */
typedef struct pa_block_manager pa_block_manager;

/* Chained hash of one block for prefix caching: FNV-1a over the block's
 * token ids started from the parent block's hash (pa_prefix_hash_seed() for
 * the first block) and mixed with it again. */
uint64_t pa_prefix_block_hash(uint64_t parent_hash, const int32_t* token_ids,
                              int num_tokens);
uint64_t pa_prefix_hash_seed(void);

/* A manager over num_blocks GPU blocks and num_cpu_blocks CPU blocks of
 * block_size tokens.  NULL on bad arguments or allocation failure.  With
 * enable_prefix_caching, every full block of a sequence whose token ids are
 * known is registered under its chained hash; a freed registered block stays
 * reusable until the allocator hands it out again (oldest first). */
pa_block_manager* pa_bm_create(int num_blocks, int num_cpu_blocks,
                               int block_size, int enable_prefix_caching);
void pa_bm_destroy(pa_block_manager* m);
int pa_bm_num_free_blocks(const pa_block_manager* m);
int pa_bm_num_free_cpu_blocks(const pa_block_manager* m);

/* New sequence holding the prompt token_ids[0..num_tokens).  With prefix
 * caching, leading full blocks whose chained hash and token ids match a
 * registered block are shared instead of allocated; *num_cached_tokens (if
 * non-NULL) gets their token count c.  slot_mapping (nullable, host,
 * num_tokens - c entries) receives the slots of tokens c..num_tokens-1, the
 * ones whose K/V the caller must write.  Returns the sequence id (>= 0),
 * PA_ERR_NO_BLOCKS (nothing changed) or PA_ERR_INVALID_ARG. */
int pa_bm_add_sequence(pa_block_manager* m, const int32_t* token_ids,
                       int num_tokens, int64_t* slot_mapping,
                       int* num_cached_tokens);

/* New sequence sharing every block of `parent` (reference counts + 1):
 * parallel sampling / beam branches.  Returns its id or a negative status. */
int pa_bm_fork(pa_block_manager* m, int parent);

/* Reserve slots for num_new_tokens tokens at the end of sequence seq_id:
 * slot_mapping (host, num_new_tokens entries) gets their slots.  Blocks are
 * allocated on demand; if the sequence's partial last block is shared, it is
 * first replaced by a fresh copy and the pair (old, new) is written to
 * cow_pairs (host int64 [cow_capacity][2]) for pa_copy_blocks, with the count
 * in *num_cow.  token_ids (nullable) feed prefix caching; once a call passes
 * NULL, the sequence's later blocks are not registered.  Returns PA_OK,
 * PA_ERR_NO_BLOCKS (nothing changed) or PA_ERR_INVALID_ARG. */
int pa_bm_append_slots(pa_block_manager* m, int seq_id, int num_new_tokens,
                       const int32_t* token_ids, int64_t* slot_mapping,
                       int64_t* cow_pairs, int cow_capacity, int* num_cow);

/* Finish a sequence: its blocks' reference counts drop, unshared blocks go
 * back to the free pool.  Returns PA_OK or PA_ERR_INVALID_ARG. */
int pa_bm_free_sequence(pa_block_manager* m, int seq_id);

/* Tokens held by the sequence, or a negative status. */
int pa_bm_seq_len(const pa_block_manager* m, int seq_id);

/* Copy the sequence's block table (physical ids, logical order) into out
 * (nullable, capacity entries).  Returns the number of blocks. */
int pa_bm_block_table(const pa_block_manager* m, int seq_id, int32_t* out,
                      int capacity);

/* Reference count of a GPU block (0 = free). */
int pa_bm_block_refcount(const pa_block_manager* m, int block);

/* Preemption by swapping: move every block of an unshared sequence to the CPU
 * pool (pa_bm_swap_out) or back to fresh GPU blocks (pa_bm_swap_in).  pairs
 * (host int64 [capacity][2]) receives the (src, dst) pairs for
 * pa_swap_blocks.  Returns the pair count or a negative status
 * (PA_ERR_INVALID_ARG if a block is shared or the sequence is already there). */
int pa_bm_swap_out(pa_block_manager* m, int seq_id, int64_t* pairs,
                   int capacity);
int pa_bm_swap_in(pa_block_manager* m, int seq_id, int64_t* pairs,
                  int capacity);

/* Shared-prefix groups of a batch, for pa_decode_attention_shared_prefix
 * ("Memory Sharing via Copy-on-Write (CoW)": parallel samples and beams share
 * the prompt's blocks until they diverge).  seq_ids (host int32
 * [num_seqs]) is the batch in launch order; runs of consecutive sequences
 * whose block tables agree on at least min_shared_blocks (>= 1) leading
 * blocks form a group, whose prefix is the blocks all its members share
 * (times block_size tokens); a sequence sharing nothing is a group of one
 * with prefix 0.  Writes group_start (host int32 [num_seqs + 1]),
 * prefix_lens (host int32 [num_seqs]) and, if non-NULL, the largest group
 * size; returns the group count, or PA_ERR_INVALID_ARG for an unknown or
 * swapped-out sequence. */
int pa_bm_shared_prefix_groups(const pa_block_manager* m, const int32_t* seq_ids,
                               int num_seqs, int min_shared_blocks,
                               int32_t* group_start, int32_t* prefix_lens,
                               int* max_group_size);

/* Capacity, in bytes, of the workspace built into the library for
 * pa_decode_attention_static_ws (32 MiB per GPU that uses the library). */
#define PA_STATIC_WORKSPACE_BYTES (32u << 20)

/*
 * pa_decode_attention_static_ws - pa_decode_attention for callers that cannot
 * allocate device memory.  The pages have no counterpart of this call: it is
 * an interface addition of this library.
 *
 * Some callers are given only their inputs and outputs and may not allocate
 * on the device themselves (plugin hooks of inference runtimes, processes
 * whose device memory another allocator reserved at start-up, C code without
 * a device allocator).  This call takes the same arguments as
 * pa_decode_attention minus the workspace, and uses as split-KV scratch a
 * fixed array of PA_STATIC_WORKSPACE_BYTES compiled into the library (held on
 * every GPU that uses the library until the process exits).  It never calls
 * cudaMalloc, cudaFree or any allocating routine.
 *
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, which allocates nothing), so the address stays
 *     right after a context has been torn down and created again.  The
 *     array itself is committed on a device when the library's device code
 *     is first loaded there (with CUDA's lazy loading, typically the first
 *     call of this function on that device); a process whose device memory
 *     another allocator reserves at start-up should make one call with
 *     num_seqs = 0 first, which commits the array and enqueues nothing.
 *     Make that first call before any stream capture.
 *   - out and the other buffers must be on the current device.
 *   - If pa_decode_workspace_size(...) for these arguments exceeds
 *     PA_STATIC_WORKSPACE_BYTES the call returns PA_ERR_WORKSPACE and
 *     enqueues nothing (use a larger partition_size, or pa_decode_attention
 *     with your own workspace).
 *   - Every call shares the one array, which keeps the last call's contents;
 *     the kernels write each scratch value before reading it, so nothing needs
 *     clearing.  Calls that overlap on the GPU (several streams, several host
 *     threads) race on the array: serialise them.
 * Other arguments, results and errors are those of pa_decode_attention.
 */
int pa_decode_attention_static_ws(float* out, const void* q,
                                  const void* k_cache, const void* v_cache,
                                  const int32_t* block_tables,
                                  int max_blocks_per_seq,
                                  const int32_t* context_lens,
                                  int max_context_len, int num_seqs,
                                  int num_heads, int num_kv_heads,
                                  int head_size, int block_size,
                                  int num_blocks, float scale,
                                  int partition_size, int* error_flags,
                                  pa_stream_t stream);

/*
 * pa_copy_blocks - copy-on-write block copies ("Memory Sharing via
 * Copy-on-Write (CoW)": when sequences sharing a block diverge, only that
 * block is copied).  For each pair p and each layer l:
 *     k_caches[l][dst] = k_caches[l][src],  v_caches[l][dst] = v_caches[l][src]
 * with (src, dst) = (block_mapping[2p], block_mapping[2p+1]); whole blocks,
 * bit-exact.
 *
 *   k_caches, v_caches   HOST arrays of num_layers device pointers, each a
 *                        pool with the layout above (same shape per layer).
 *   block_mapping        int64 [num_pairs][2], device.
 *   num_pairs            >= 0 (0 enqueues nothing).
 *   error_flags          nullable device int; PA_DEVERR_COPY_PAIR on an id
 *                        outside [0, num_blocks) (that pair is skipped).
 * Pairs run concurrently, so no dst may equal another pair's src or dst
 * (src == dst is a no-op); a mapping that breaks this has an unspecified
 * result.  Returns PA_OK or a negative pa_status.
 */
int pa_copy_blocks(void* const* k_caches, void* const* v_caches,
                   int num_layers, const int64_t* block_mapping, int num_pairs,
                   int num_blocks, int block_size, int num_kv_heads,
                   int head_size, int* error_flags, pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_B200_PA_H */
