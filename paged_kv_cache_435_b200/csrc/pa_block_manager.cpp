// Host-side KV block manager: the bookkeeping that feeds the kernels.
//
//  * A free pool of physical blocks (a FIFO queue; freed blocks go to the
//    back, allocation takes the front) and, per sequence, a block table of
//    logical -> physical ids.  Blocks are allocated on demand as a sequence
//    grows ("vLLM: Anatomy and Mechanisms of High-Throughput LLM Inference",
//    "Block-Level Management"; "Inside vLLM: Anatomy of a High-Throughput LLM
//    Inference System", KV-cache manager's free_block_queue and
//    allocate_slots; "vLLM Internals", "The Block Manager").
//  * Sharing with reference counts: a forked sequence (parallel sampling,
//    beams) points at its parent's blocks; writing into a shared block first
//    copies that one block (copy-on-write, "Memory Sharing via Copy-on-Write
//    (CoW)"), and the (src, dst) pair is handed to pa_copy_blocks.
//  * Prefix caching: every full block gets a hash chained from the previous
//    block's hash and its own token ids; a new prompt whose leading blocks hash
//    the same reuses them ("Prefix Caching": chunks of 16 tokens are hashed and
//    matching blocks reused).  Freed hashed blocks stay findable until the
//    allocator hands them out again, oldest first.  A hit also compares the
//    stored token ids, so a hash collision can never alias two prefixes.
//  * Swapping: a sequence's blocks can move to a CPU pool and back, producing
//    the (src, dst) pairs for pa_swap_blocks ("Preemption and Recovery").
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"

namespace {

constexpr uint64_t kHashSeed = 0xcbf29ce484222325ull;  // FNV-1a offset basis
constexpr uint64_t kHashPrime = 0x100000001b3ull;      // FNV-1a prime

uint64_t fnv1a(uint64_t h, const void* data, size_t n) {
    const unsigned char* p = static_cast<const unsigned char*>(data);
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= kHashPrime;
    }
    return h;
}

struct Pool {
    // Per physical block.
    std::vector<int> ref;
    std::vector<int> prev, next;       // free-queue links (-1 = none)
    std::vector<char> in_free;
    std::vector<char> hashed;
    std::vector<uint64_t> hash;
    std::vector<int32_t> tokens;       // block_size ids per hashed block
    int head = -1, tail = -1, free_count = 0;

    void init(int n) {
        ref.assign(n, 0);
        prev.assign(n, -1);
        next.assign(n, -1);
        in_free.assign(n, 0);
        hashed.assign(n, 0);
        hash.assign(n, 0);
        head = tail = -1;
        free_count = 0;
        for (int b = 0; b < n; ++b) push_back(b);
    }
    void push_back(int b) {
        prev[b] = tail;
        next[b] = -1;
        if (tail >= 0) next[tail] = b; else head = b;
        tail = b;
        in_free[b] = 1;
        ++free_count;
    }
    void unlink(int b) {
        if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
        if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
        prev[b] = next[b] = -1;
        in_free[b] = 0;
        --free_count;
    }
};

struct Sequence {
    bool alive = false;
    bool on_cpu = false;
    bool hashing = true;               // token ids known for every block so far
    std::vector<int> blocks;           // block table (GPU or CPU ids)
    int len = 0;                       // tokens held
    std::vector<int32_t> tail_tokens;  // token ids of the partial last block
    uint64_t last_full_hash = kHashSeed;
};

}  // namespace

extern "C" uint64_t pa_prefix_block_hash(uint64_t parent_hash,
                                         const int32_t* token_ids,
                                         int num_tokens);

struct pa_block_manager {
    int num_blocks = 0, num_cpu_blocks = 0, block_size = 0;
    bool prefix_caching = false;
    Pool gpu, cpu;
    std::unordered_map<uint64_t, int> cached;  // hash -> GPU block
    std::vector<Sequence> seqs;

    int alloc_gpu() {
        const int b = gpu.head;
        if (b < 0) return -1;
        gpu.unlink(b);
        if (gpu.hashed[b]) {  // evict its cache entry
            auto it = cached.find(gpu.hash[b]);
            if (it != cached.end() && it->second == b) cached.erase(it);
            gpu.hashed[b] = 0;
        }
        gpu.ref[b] = 1;
        return b;
    }
    void release_gpu(int b) {
        if (--gpu.ref[b] == 0) gpu.push_back(b);
    }
    // Register a just-filled block under its chained hash.
    void register_full(Sequence& s, int b, const int32_t* toks) {
        const uint64_t h = pa_prefix_block_hash(s.last_full_hash, toks, block_size);
        s.last_full_hash = h;
        if (!prefix_caching || gpu.hashed[b]) return;
        if (cached.count(h)) return;  // an identical block is already cached
        gpu.hashed[b] = 1;
        gpu.hash[b] = h;
        std::memcpy(&gpu.tokens[(size_t)b * block_size], toks,
                    sizeof(int32_t) * (size_t)block_size);
        cached[h] = b;
    }
    int find_cached(uint64_t h, const int32_t* toks) const {
        auto it = cached.find(h);
        if (it == cached.end()) return -1;
        const int b = it->second;
        if (std::memcmp(&gpu.tokens[(size_t)b * block_size], toks,
                        sizeof(int32_t) * (size_t)block_size) != 0)
            return -1;
        return b;
    }
    Sequence* seq(int id) {
        if (id < 0 || id >= (int)seqs.size() || !seqs[id].alive) return nullptr;
        return &seqs[id];
    }
    int new_seq_id() {
        for (int i = 0; i < (int)seqs.size(); ++i)
            if (!seqs[i].alive) return i;
        seqs.emplace_back();
        return (int)seqs.size() - 1;
    }
};

extern "C" {

// FNV-1a over the block's token ids, started from the parent block's hash and
// mixed with it once more, so equal blocks under different prefixes differ.
uint64_t pa_prefix_block_hash(uint64_t parent_hash, const int32_t* token_ids,
                              int num_tokens) {
    if (num_tokens < 0 || (num_tokens > 0 && !token_ids)) return 0;
    return fnv1a(parent_hash, token_ids, sizeof(int32_t) * (size_t)num_tokens) ^
           (parent_hash * kHashPrime);
}

uint64_t pa_prefix_hash_seed(void) { return kHashSeed; }

pa_block_manager* pa_bm_create(int num_blocks, int num_cpu_blocks,
                               int block_size, int enable_prefix_caching) {
    if (num_blocks <= 0 || num_cpu_blocks < 0 || block_size <= 0) return nullptr;
    pa_block_manager* m = new (std::nothrow) pa_block_manager();
    if (!m) return nullptr;
    try {
        m->num_blocks = num_blocks;
        m->num_cpu_blocks = num_cpu_blocks;
        m->block_size = block_size;
        m->prefix_caching = enable_prefix_caching != 0;
        m->gpu.init(num_blocks);
        m->gpu.tokens.assign((size_t)num_blocks * block_size, 0);
        m->cpu.init(num_cpu_blocks);
    } catch (...) {
        delete m;
        return nullptr;
    }
    return m;
}

void pa_bm_destroy(pa_block_manager* m) { delete m; }

int pa_bm_num_free_blocks(const pa_block_manager* m) {
    return m ? m->gpu.free_count : PA_ERR_INVALID_ARG;
}

int pa_bm_num_free_cpu_blocks(const pa_block_manager* m) {
    return m ? m->cpu.free_count : PA_ERR_INVALID_ARG;
}

int pa_bm_add_sequence(pa_block_manager* m, const int32_t* token_ids,
                       int num_tokens, int64_t* slot_mapping,
                       int* num_cached_tokens) {
    if (!m || num_tokens < 0 || (num_tokens > 0 && !token_ids)) return PA_ERR_INVALID_ARG;
    try {
        const int bs = m->block_size;
        const int id = m->new_seq_id();
        Sequence s;
        s.alive = true;
        // Reuse cached full blocks of the prompt's prefix.
        int reused = 0;
        uint64_t h = kHashSeed;
        if (m->prefix_caching) {
            for (int i = 0; (i + 1) * bs <= num_tokens; ++i) {
                const int32_t* toks = token_ids + (size_t)i * bs;
                const uint64_t hi = pa_prefix_block_hash(h, toks, bs);
                const int b = m->find_cached(hi, toks);
                if (b < 0) break;
                if (m->gpu.in_free[b]) m->gpu.unlink(b);
                ++m->gpu.ref[b];
                s.blocks.push_back(b);
                h = hi;
                ++reused;
            }
        }
        const int need = (num_tokens + bs - 1) / bs - reused;
        if (need > m->gpu.free_count) {
            for (int b : s.blocks) m->release_gpu(b);
            return PA_ERR_NO_BLOCKS;
        }
        s.last_full_hash = h;
        s.len = reused * bs;
        for (int t = s.len; t < num_tokens; ++t) {
            if (t % bs == 0) s.blocks.push_back(m->alloc_gpu());
            const int b = s.blocks[t / bs];
            if (slot_mapping) slot_mapping[t - reused * bs] = (int64_t)b * bs + t % bs;
            s.tail_tokens.push_back(token_ids[t]);
            ++s.len;
            if (s.len % bs == 0) {
                m->register_full(s, b, s.tail_tokens.data());
                s.tail_tokens.clear();
            }
        }
        if (num_cached_tokens) *num_cached_tokens = reused * bs;
        m->seqs[id] = std::move(s);
        return id;
    } catch (...) {
        return PA_ERR_NO_BLOCKS;
    }
}

int pa_bm_fork(pa_block_manager* m, int parent) {
    if (!m || !m->seq(parent) || m->seqs[parent].on_cpu) return PA_ERR_INVALID_ARG;
    try {
        const int id = m->new_seq_id();
        Sequence child = m->seqs[parent];
        for (int b : child.blocks) ++m->gpu.ref[b];
        m->seqs[id] = std::move(child);
        return id;
    } catch (...) {
        return PA_ERR_NO_BLOCKS;
    }
}

int pa_bm_append_slots(pa_block_manager* m, int seq_id, int num_new_tokens,
                       const int32_t* token_ids, int64_t* slot_mapping,
                       int64_t* cow_pairs, int cow_capacity, int* num_cow) {
    if (!m || num_new_tokens < 0 || !slot_mapping || cow_capacity < 0)
        return PA_ERR_INVALID_ARG;
    Sequence* s = m->seq(seq_id);
    if (!s || s->on_cpu) return PA_ERR_INVALID_ARG;
    const int bs = m->block_size;
    // Blocks this call may need: new ones plus one copy of a shared tail.
    const int new_blocks = (s->len + num_new_tokens + bs - 1) / bs - (s->len + bs - 1) / bs;
    const bool tail_shared = s->len % bs != 0 && num_new_tokens > 0 &&
                             m->gpu.ref[s->blocks.back()] > 1;
    if (new_blocks + (tail_shared ? 1 : 0) > m->gpu.free_count) return PA_ERR_NO_BLOCKS;
    if (tail_shared && cow_capacity < 1) return PA_ERR_INVALID_ARG;
    int cows = 0;
    for (int i = 0; i < num_new_tokens; ++i) {
        const int t = s->len;
        if (t % bs == 0) {
            s->blocks.push_back(m->alloc_gpu());
        } else if (m->gpu.ref[s->blocks.back()] > 1) {
            // Copy-on-write: this sequence diverges inside a shared block.
            const int old = s->blocks.back();
            const int fresh = m->alloc_gpu();
            m->release_gpu(old);
            s->blocks.back() = fresh;
            cow_pairs[2 * cows] = old;
            cow_pairs[2 * cows + 1] = fresh;
            ++cows;
        }
        const int b = s->blocks[t / bs];
        slot_mapping[i] = (int64_t)b * bs + t % bs;
        if (!token_ids) s->hashing = false;  // later blocks cannot be hashed
        s->tail_tokens.push_back(token_ids ? token_ids[i] : 0);
        ++s->len;
        if (s->len % bs == 0) {
            if (s->hashing) m->register_full(*s, b, s->tail_tokens.data());
            s->tail_tokens.clear();
        }
    }
    if (num_cow) *num_cow = cows;
    return PA_OK;
}

int pa_bm_free_sequence(pa_block_manager* m, int seq_id) {
    Sequence* s = m ? m->seq(seq_id) : nullptr;
    if (!s) return PA_ERR_INVALID_ARG;
    if (s->on_cpu) {
        for (int b : s->blocks) m->cpu.push_back(b);
    } else {
        // Release in reverse so the tail (least shareable) is reused first.
        for (int i = (int)s->blocks.size() - 1; i >= 0; --i) m->release_gpu(s->blocks[i]);
    }
    *s = Sequence();
    return PA_OK;
}

int pa_bm_seq_len(const pa_block_manager* m, int seq_id) {
    if (!m || seq_id < 0 || seq_id >= (int)m->seqs.size() || !m->seqs[seq_id].alive)
        return PA_ERR_INVALID_ARG;
    return m->seqs[seq_id].len;
}

int pa_bm_block_table(const pa_block_manager* m, int seq_id, int32_t* out,
                      int capacity) {
    if (!m || seq_id < 0 || seq_id >= (int)m->seqs.size() || !m->seqs[seq_id].alive)
        return PA_ERR_INVALID_ARG;
    const std::vector<int>& b = m->seqs[seq_id].blocks;
    if (out) {
        if (capacity < (int)b.size()) return PA_ERR_INVALID_ARG;
        for (size_t i = 0; i < b.size(); ++i) out[i] = b[i];
    }
    return (int)b.size();
}

int pa_bm_block_refcount(const pa_block_manager* m, int block) {
    if (!m || block < 0 || block >= m->num_blocks) return PA_ERR_INVALID_ARG;
    return m->gpu.ref[block];
}

int pa_bm_swap_out(pa_block_manager* m, int seq_id, int64_t* pairs,
                   int capacity) {
    Sequence* s = m ? m->seq(seq_id) : nullptr;
    if (!s || s->on_cpu || !pairs) return PA_ERR_INVALID_ARG;
    const int n = (int)s->blocks.size();
    if (capacity < n) return PA_ERR_INVALID_ARG;
    for (int b : s->blocks)
        if (m->gpu.ref[b] != 1) return PA_ERR_INVALID_ARG;  // shared: not movable alone
    if (n > m->cpu.free_count) return PA_ERR_NO_BLOCKS;
    for (int i = 0; i < n; ++i) {
        const int c = m->cpu.head;
        m->cpu.unlink(c);
        pairs[2 * i] = s->blocks[i];
        pairs[2 * i + 1] = c;
        m->release_gpu(s->blocks[i]);
        s->blocks[i] = c;
    }
    s->on_cpu = true;
    return n;
}

int pa_bm_swap_in(pa_block_manager* m, int seq_id, int64_t* pairs,
                  int capacity) {
    Sequence* s = m ? m->seq(seq_id) : nullptr;
    if (!s || !s->on_cpu || !pairs) return PA_ERR_INVALID_ARG;
    const int n = (int)s->blocks.size();
    if (capacity < n) return PA_ERR_INVALID_ARG;
    if (n > m->gpu.free_count) return PA_ERR_NO_BLOCKS;
    for (int i = 0; i < n; ++i) {
        const int g = m->alloc_gpu();
        pairs[2 * i] = s->blocks[i];
        pairs[2 * i + 1] = g;
        m->cpu.push_back(s->blocks[i]);
        s->blocks[i] = g;
    }
    s->on_cpu = false;
    return n;
}

// Groups for pa_decode_attention_shared_prefix: runs of consecutive batch
// sequences whose block tables agree on at least min_shared_blocks leading
// blocks; a group's prefix is the blocks all its members share.
int pa_bm_shared_prefix_groups(const pa_block_manager* m, const int32_t* seq_ids,
                               int num_seqs, int min_shared_blocks,
                               int32_t* group_start, int32_t* prefix_lens,
                               int* max_group_size) {
    if (!m || num_seqs < 0 || min_shared_blocks < 1) return PA_ERR_INVALID_ARG;
    if (!group_start || (num_seqs > 0 && (!seq_ids || !prefix_lens)))
        return PA_ERR_INVALID_ARG;
    for (int i = 0; i < num_seqs; ++i) {
        const int id = seq_ids[i];
        if (id < 0 || id >= (int)m->seqs.size() || !m->seqs[id].alive ||
            m->seqs[id].on_cpu)
            return PA_ERR_INVALID_ARG;
    }
    int groups = 0, largest = 1;
    group_start[0] = 0;
    for (int i = 0; i < num_seqs;) {
        const std::vector<int>& first = m->seqs[seq_ids[i]].blocks;
        int common = (int)first.size();
        int j = i + 1;
        for (; j < num_seqs; ++j) {
            const std::vector<int>& b = m->seqs[seq_ids[j]].blocks;
            const int lim = std::min(common, (int)b.size());
            int c = 0;
            while (c < lim && b[c] == first[c]) ++c;
            if (c < min_shared_blocks) break;
            common = c;
        }
        // A sequence alone shares nothing: it gets the per-sequence pass only.
        prefix_lens[groups] = j - i >= 2 ? common * m->block_size : 0;
        group_start[++groups] = j;
        largest = std::max(largest, j - i);
        i = j;
    }
    if (max_group_size) *max_group_size = largest;
    return groups;
}

}  // extern "C"
