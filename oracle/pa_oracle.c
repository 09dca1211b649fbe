/*
 * Plain fp64 CPU oracle for paged decode attention and its two cache
 * companions.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline arm may call it; the product path never does.  It
 * shares no code, header or constant with the CUDA library.
 *
 * What it computes, and where the method is described:
 *
 *  - Paged KV pool.  Each layer's K and V caches are arrays of fixed-size
 *    physical blocks, [num_blocks][block_size][num_kv_heads][head_size] in
 *    bf16.  A sequence's logical token t lives in physical block
 *    block_table[t / block_size] at offset t % block_size.
 *    ("vLLM: Anatomy and Mechanisms of High-Throughput LLM Inference",
 *    section "PagedAttention: The vLLM Innovation" / "Block-Level
 *    Management"; per-block byte count 2*block_size*num_kv_heads*head_size*
 *    dtype_bytes from "Inside vLLM: Anatomy of a High-Throughput LLM
 *    Inference System", section "LLM Engine constructor", KV-cache manager.)
 *
 *  - Decode attention.  One query token per sequence attends over the
 *    sequence's whole cached context (decode step, "Prefill vs. Decode
 *    Operations" of the first page).  For query head h the kv head is
 *    h / (num_heads / num_kv_heads) (contiguous grouping; the pages name only
 *    num_kv_heads, this is the reading taken).  Logits z_t = scale * q.k_t,
 *    weights softmax(z), output sum_t w_t v_t.  No partitioning, no online
 *    rescaling: the definition, evaluated directly in double precision.
 *
 *  - reshape_and_cache.  Token i's new K/V rows go to slot s = slot_mapping[i]
 *    (block s / block_size, offset s % block_size); a negative slot is padding
 *    and is skipped.  (On-demand block allocation, "Block-Level Management";
 *    "Allocate, reshape and bind KV cache tensors", second page.)
 *
 *  - copy_blocks.  Copy-on-write: each (src, dst) pair copies the whole
 *    physical block, K and V, in every layer ("Memory Sharing via
 *    Copy-on-Write (CoW)" of the first page).
 *
 * bf16 values are widened exactly (bf16 is the upper half of an IEEE binary32).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_RANGE (-2)
#define ORACLE_ERR_NOMEM (-3)

static double bf16_bits_to_double(uint16_t bits) {
    uint32_t word = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &word, sizeof f);
    return (double)f;
}

/* Flat index of element [blk][off][head][d] of a pool shaped
 * [num_blocks][block_size][num_kv_heads][head_size]. */
static int64_t pool_index(int64_t blk, int64_t off, int64_t head, int64_t d,
                          int64_t block_size, int64_t num_kv_heads,
                          int64_t head_size) {
    return ((blk * block_size + off) * num_kv_heads + head) * head_size + d;
}

/* ------------------------------------------------------------------------ */
/* reshape_and_cache                                                          */
/* ------------------------------------------------------------------------ */
int oracle_reshape_and_cache(const uint16_t* key, const uint16_t* value,
                             int64_t key_token_stride,
                             int64_t value_token_stride, uint16_t* k_cache,
                             uint16_t* v_cache, const int64_t* slot_mapping,
                             int num_tokens, int num_blocks, int block_size,
                             int num_kv_heads, int head_size) {
    if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 ||
        num_kv_heads <= 0 || head_size <= 0)
        return ORACLE_ERR_ARG;
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0) continue; /* padding token */
        int64_t blk = slot / block_size;
        int64_t off = slot % block_size;
        if (blk >= num_blocks) return ORACLE_ERR_RANGE;
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int d = 0; d < head_size; ++d) {
                int64_t dst = pool_index(blk, off, h, d, block_size,
                                         num_kv_heads, head_size);
                k_cache[dst] = key[(int64_t)i * key_token_stride +
                                   (int64_t)h * head_size + d];
                v_cache[dst] = value[(int64_t)i * value_token_stride +
                                     (int64_t)h * head_size + d];
            }
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* copy_blocks                                                                */
/* ------------------------------------------------------------------------ */
int oracle_copy_blocks(uint16_t* const* k_caches, uint16_t* const* v_caches,
                       int num_layers, const int64_t* block_mapping,
                       int num_pairs, int num_blocks, int block_size,
                       int num_kv_heads, int head_size) {
    if (num_layers <= 0 || num_pairs < 0 || num_blocks <= 0 ||
        block_size <= 0 || num_kv_heads <= 0 || head_size <= 0)
        return ORACLE_ERR_ARG;
    size_t block_elems = (size_t)block_size * num_kv_heads * head_size;
    for (int p = 0; p < num_pairs; ++p) {
        int64_t src = block_mapping[2 * p];
        int64_t dst = block_mapping[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks)
            return ORACLE_ERR_RANGE;
        for (int layer = 0; layer < num_layers; ++layer) {
            memmove(k_caches[layer] + dst * block_elems,
                    k_caches[layer] + src * block_elems,
                    block_elems * sizeof(uint16_t));
            memmove(v_caches[layer] + dst * block_elems,
                    v_caches[layer] + src * block_elems,
                    block_elems * sizeof(uint16_t));
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* paged decode attention                                                     */
/* ------------------------------------------------------------------------ */
typedef struct {
    double* out;
    const uint16_t* q;
    const uint16_t* k_cache;
    const uint16_t* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    int max_blocks_per_seq, num_seqs, num_heads, num_kv_heads, head_size;
    int block_size, num_blocks;
    double scale;
    int next_item; /* shared work counter, guarded by lock */
    pthread_mutex_t lock;
    int status;
} attn_job;

/* out[s][h][:] for one (sequence, query head). */
static int attend_one(attn_job* job, int s, int h) {
    const int D = job->head_size;
    const int G = job->num_heads / job->num_kv_heads;
    const int kv = h / G;
    const int L = job->context_lens[s];
    double* o = job->out + ((int64_t)s * job->num_heads + h) * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (L <= 0) return ORACLE_OK; /* empty context: zeros */
    if (L > job->max_blocks_per_seq * job->block_size) return ORACLE_ERR_RANGE;

    const uint16_t* qv = job->q + ((int64_t)s * job->num_heads + h) * D;
    double* z = (double*)malloc(sizeof(double) * (size_t)L);
    if (!z) return ORACLE_ERR_NOMEM;

    /* z_t = scale * sum_d q[d] k_t[d], k_t gathered through the block table */
    for (int t = 0; t < L; ++t) {
        int32_t phys = job->block_tables[(int64_t)s * job->max_blocks_per_seq +
                                         t / job->block_size];
        int off = t % job->block_size;
        if (phys < 0 || phys >= job->num_blocks) {
            free(z);
            return ORACLE_ERR_RANGE;
        }
        double dot = 0.0;
        for (int d = 0; d < D; ++d) {
            int64_t idx = pool_index(phys, off, kv, d, job->block_size,
                                     job->num_kv_heads, D);
            dot += bf16_bits_to_double(qv[d]) *
                   bf16_bits_to_double(job->k_cache[idx]);
        }
        z[t] = job->scale * dot;
    }

    /* softmax weights w_t = exp(z_t - max z) / sum */
    double zmax = z[0];
    for (int t = 1; t < L; ++t)
        if (z[t] > zmax) zmax = z[t];
    double wsum = 0.0;
    for (int t = 0; t < L; ++t) {
        z[t] = exp(z[t] - zmax);
        wsum += z[t];
    }

    /* out = sum_t w_t v_t / sum_t w_t */
    for (int t = 0; t < L; ++t) {
        int32_t phys = job->block_tables[(int64_t)s * job->max_blocks_per_seq +
                                         t / job->block_size];
        int off = t % job->block_size;
        for (int d = 0; d < D; ++d) {
            int64_t idx = pool_index(phys, off, kv, d, job->block_size,
                                     job->num_kv_heads, D);
            o[d] += z[t] * bf16_bits_to_double(job->v_cache[idx]);
        }
    }
    for (int d = 0; d < D; ++d) o[d] /= wsum;
    free(z);
    return ORACLE_OK;
}

static void* attn_worker(void* arg) {
    attn_job* job = (attn_job*)arg;
    const int total = job->num_seqs * job->num_heads;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        int item = job->next_item++;
        int failed = job->status != ORACLE_OK;
        pthread_mutex_unlock(&job->lock);
        if (item >= total || failed) break;
        int rc = attend_one(job, item / job->num_heads, item % job->num_heads);
        if (rc != ORACLE_OK) {
            pthread_mutex_lock(&job->lock);
            if (job->status == ORACLE_OK) job->status = rc;
            pthread_mutex_unlock(&job->lock);
        }
    }
    return NULL;
}

/* Output: double out[num_seqs][num_heads][head_size].  The (sequence, head)
 * pairs are independent; num_threads > 1 spreads them over POSIX threads
 * without changing any arithmetic. */
int oracle_paged_decode_attention(
    double* out, const uint16_t* q, const uint16_t* k_cache,
    const uint16_t* v_cache, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
    int num_heads, int num_kv_heads, int head_size, int block_size,
    int num_blocks, double scale, int num_threads) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        head_size <= 0 || block_size <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || num_heads % num_kv_heads != 0)
        return ORACLE_ERR_ARG;
    attn_job job;
    job.out = out;
    job.q = q;
    job.k_cache = k_cache;
    job.v_cache = v_cache;
    job.block_tables = block_tables;
    job.context_lens = context_lens;
    job.max_blocks_per_seq = max_blocks_per_seq;
    job.num_seqs = num_seqs;
    job.num_heads = num_heads;
    job.num_kv_heads = num_kv_heads;
    job.head_size = head_size;
    job.block_size = block_size;
    job.num_blocks = num_blocks;
    job.scale = scale;
    job.next_item = 0;
    job.status = ORACLE_OK;
    pthread_mutex_init(&job.lock, NULL);

    if (num_threads < 1) num_threads = 1;
    if (num_threads > 256) num_threads = 256;
    pthread_t tids[256];
    int started = 0;
    for (int i = 1; i < num_threads; ++i) {
        if (pthread_create(&tids[started], NULL, attn_worker, &job) != 0) break;
        ++started;
    }
    attn_worker(&job); /* the calling thread works too */
    for (int i = 0; i < started; ++i) pthread_join(tids[i], NULL);
    pthread_mutex_destroy(&job.lock);
    return job.status;
}

/* ------------------------------------------------------------------------ */
/* multi-query paged attention (chunked prefill / speculative verification)  */
/* ------------------------------------------------------------------------ */
/* Sequence s holds L = context_lens[s] cached tokens, of which the last
 * k = query_start_loc[s+1] - query_start_loc[s] are the new query tokens
 * (their K/V already written).  Query token j (0 <= j < k) sits at logical
 * position L - k + j and attends causally to tokens t <= L - k + j
 * ("vLLM: Anatomy and Mechanisms of High-Throughput LLM Inference",
 * "Chunked Prefill" and "Speculative Decoding": the large model verifies all
 * k proposed tokens in one forward pass).  q and out are indexed by the
 * global query token query_start_loc[s] + j.  Output double
 * out[num_q_tokens][num_heads][head_size]. */
typedef struct {
    double* out;
    const uint16_t* q;
    const uint16_t* k_cache;
    const uint16_t* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start_loc;
    int max_blocks_per_seq, num_seqs, num_heads, num_kv_heads, head_size;
    int block_size, num_blocks;
    double scale;
    int next_item;
    pthread_mutex_t lock;
    int status;
} mq_job;

static int mq_attend_one(mq_job* job, int s, int h) {
    const int D = job->head_size;
    const int G = job->num_heads / job->num_kv_heads;
    const int kv = h / G;
    const int L = job->context_lens[s];
    const int q0 = job->query_start_loc[s];
    const int k = job->query_start_loc[s + 1] - q0;
    if (k < 0 || k > L || L > job->max_blocks_per_seq * job->block_size)
        return ORACLE_ERR_RANGE;
    double* z = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    if (!z) return ORACLE_ERR_NOMEM;
    for (int j = 0; j < k; ++j) {
        const int last = L - k + j; /* last visible logical position */
        const uint16_t* qv = job->q + ((int64_t)(q0 + j) * job->num_heads + h) * D;
        double* o = job->out + ((int64_t)(q0 + j) * job->num_heads + h) * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        for (int t = 0; t <= last; ++t) {
            int32_t phys = job->block_tables[(int64_t)s * job->max_blocks_per_seq +
                                             t / job->block_size];
            if (phys < 0 || phys >= job->num_blocks) {
                free(z);
                return ORACLE_ERR_RANGE;
            }
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += bf16_bits_to_double(qv[d]) *
                       bf16_bits_to_double(job->k_cache[pool_index(
                           phys, t % job->block_size, kv, d, job->block_size,
                           job->num_kv_heads, D)]);
            z[t] = job->scale * dot;
        }
        double zmax = z[0];
        for (int t = 1; t <= last; ++t)
            if (z[t] > zmax) zmax = z[t];
        double wsum = 0.0;
        for (int t = 0; t <= last; ++t) {
            z[t] = exp(z[t] - zmax);
            wsum += z[t];
        }
        for (int t = 0; t <= last; ++t) {
            int32_t phys = job->block_tables[(int64_t)s * job->max_blocks_per_seq +
                                             t / job->block_size];
            for (int d = 0; d < D; ++d)
                o[d] += z[t] * bf16_bits_to_double(job->v_cache[pool_index(
                                   phys, t % job->block_size, kv, d,
                                   job->block_size, job->num_kv_heads, D)]);
        }
        for (int d = 0; d < D; ++d) o[d] /= wsum;
    }
    free(z);
    return ORACLE_OK;
}

static void* mq_worker(void* arg) {
    mq_job* job = (mq_job*)arg;
    const int total = job->num_seqs * job->num_heads;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        int item = job->next_item++;
        int failed = job->status != ORACLE_OK;
        pthread_mutex_unlock(&job->lock);
        if (item >= total || failed) break;
        int rc = mq_attend_one(job, item / job->num_heads, item % job->num_heads);
        if (rc != ORACLE_OK) {
            pthread_mutex_lock(&job->lock);
            if (job->status == ORACLE_OK) job->status = rc;
            pthread_mutex_unlock(&job->lock);
        }
    }
    return NULL;
}

int oracle_paged_multi_query_attention(
    double* out, const uint16_t* q, const uint16_t* k_cache,
    const uint16_t* v_cache, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* context_lens,
    const int32_t* query_start_loc, int num_seqs, int num_heads,
    int num_kv_heads, int head_size, int block_size, int num_blocks,
    double scale, int num_threads) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        head_size <= 0 || block_size <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || num_heads % num_kv_heads != 0)
        return ORACLE_ERR_ARG;
    mq_job job;
    job.out = out;
    job.q = q;
    job.k_cache = k_cache;
    job.v_cache = v_cache;
    job.block_tables = block_tables;
    job.context_lens = context_lens;
    job.query_start_loc = query_start_loc;
    job.max_blocks_per_seq = max_blocks_per_seq;
    job.num_seqs = num_seqs;
    job.num_heads = num_heads;
    job.num_kv_heads = num_kv_heads;
    job.head_size = head_size;
    job.block_size = block_size;
    job.num_blocks = num_blocks;
    job.scale = scale;
    job.next_item = 0;
    job.status = ORACLE_OK;
    pthread_mutex_init(&job.lock, NULL);
    if (num_threads < 1) num_threads = 1;
    if (num_threads > 256) num_threads = 256;
    pthread_t tids[256];
    int started = 0;
    for (int i = 1; i < num_threads; ++i) {
        if (pthread_create(&tids[started], NULL, mq_worker, &job) != 0) break;
        ++started;
    }
    mq_worker(&job);
    for (int i = 0; i < started; ++i) pthread_join(tids[i], NULL);
    pthread_mutex_destroy(&job.lock);
    return job.status;
}

/* ------------------------------------------------------------------------ */
/* swap_blocks                                                                */
/* ------------------------------------------------------------------------ */
/* Preemption by swapping: evicted KV blocks are moved to CPU RAM and brought
 * back when the request is rescheduled ("vLLM: Anatomy and Mechanisms of
 * High-Throughput LLM Inference", "Preemption and Recovery"; "vLLM
 * Internals", "The Block Manager").  For each pair (src, dst) and each cache
 * c: dst_caches[c] block dst = src_caches[c] block src, block_bytes bytes. */
int oracle_swap_blocks(const uint8_t* const* src_caches, uint8_t* const* dst_caches,
                       int num_caches, const int64_t* block_mapping, int num_pairs,
                       int64_t block_bytes, int64_t src_num_blocks,
                       int64_t dst_num_blocks) {
    if (num_caches <= 0 || num_pairs < 0 || block_bytes <= 0) return ORACLE_ERR_ARG;
    for (int p = 0; p < num_pairs; ++p) {
        int64_t src = block_mapping[2 * p];
        int64_t dst = block_mapping[2 * p + 1];
        if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks)
            return ORACLE_ERR_RANGE;
        for (int c = 0; c < num_caches; ++c)
            memcpy(dst_caches[c] + dst * block_bytes,
                   src_caches[c] + src * block_bytes, (size_t)block_bytes);
    }
    return ORACLE_OK;
}
