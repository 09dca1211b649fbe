// Paged decode attention for sm_100a.
//
// The method: one new query token per sequence attends over the sequence's
// cached K/V, which live in fixed-size physical blocks found through the
// sequence's block table ("vLLM: Anatomy and Mechanisms of High-Throughput
// LLM Inference", "PagedAttention: The vLLM Innovation" / "Block-Level
// Management"; "vLLM Internals", "The Block Manager").  Decode is bound by
// the bandwidth of streaming the KV cache (first page, "Prefill vs. Decode
// Operations" and "The Roofline Model"), so the design goal is to read every
// needed KV byte exactly once at close to HBM speed.
//
// Work unit ("item"): one (sequence, KV partition) for one kv head.  A CTA of
// 4 warps processes items; warp w owns 16-token chunks w, w+4, w+8, ... of
// each item.
//  * Loads: every warp runs its own ring of shared-memory stages guarded by
//    mbarriers with transaction counts.  Lane 0 fills a stage with 2 * D/64
//    TMA tensor copies (cp.async.bulk.tensor, 128-byte swizzle): 16 rows of
//    K and of V for this kv head, 8 KB at D=128.  The producer side of the
//    ring runs ahead across item boundaries, so copies stay in flight while
//    an item is being merged.  Block ids for the next 32 chunks are
//    prefetched into one register per lane.
//  * Math: the G = num_heads/num_kv_heads query heads of the kv head share the
//    pass.  S = Q K^T and O += P V run on the bf16 tensor cores with
//    mma.m16n8k16: rows 0..7 of the 16-row M tile hold the G heads, and the
//    spare rows 8..15 carry the low-order bf16 part of P (P = P_hi + P_lo), so
//    the PV product keeps ~16 bits of P.  fp32 online softmax in the log2
//    domain; O is rescaled only when a row's running max grows.
//  * Item end: warps 1..3 post (max, sum, O) to shared memory and continue;
//    warp 0 merges and writes either the output or, when the sequence is
//    split, the partition's (max, sum, normalised O) for the merge kernel.
//  * Grids: without a split, one CTA per (kv head, sequence) item, scheduled
//    by the hardware.  With a split, a persistent grid of ~2 CTAs per SM; each
//    CTA builds the prefix sum of partitions per sequence in shared memory
//    and walks a compact item list, so no CTA is spent on partitions past a
//    sequence's end.
#include <cuda.h>

#include <cfloat>
#include <cstdint>
#include <mutex>
#include <utility>

#include "pa_common.cuh"
#include "pa_decode.cuh"

namespace pa {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 16;          // tokens per pipeline stage
constexpr int kMaxGroup = 8;
constexpr int kMaxPersistSeqs = 768;
constexpr int kTargetCtasPerSM = 2;
constexpr float kLog2e = 1.4426950408889634f;

#ifdef PA_TEST_UNSIGNALLED_FIRST_WAIT
// Test build only (libpagedattn_waittest.so, never the product library):
// every warp's first chunk wait polls a spare barrier that nothing arrives
// on, so it runs out after this limit and the kernel takes its timeout path
// (report PA_DEVERR_TIMEOUT, skip the rest, drain the copies already issued
// with the full limit).  This is how a test makes a bounded wait expire
// without any GPU fault.
constexpr unsigned long long kTestWaitLimitNs = 20000000ull;  // 20 ms
#endif

template <int D>
struct Cfg {
    static constexpr int kHalves = D / 64;                  // 128-byte column tiles
    static constexpr int kHalfBytes = kChunk * 128;         // 16 rows x 128 B
    static constexpr int kKVBytes = kHalves * kHalfBytes;   // K (or V) of a chunk
    static constexpr int kStageBytes = 2 * kKVBytes;
    static constexpr int kStages = D == 128 ? 3 : 5;
    static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
    // Item-end exchange: warps 1..3 post their partial O rows for warp 0.
    static constexpr int kRedStride = D + 8;                // floats per row
    static constexpr int kRedOBytes = (kWarps - 1) * kMaxGroup * kRedStride * 4;
    static constexpr int kRedMLBytes = kWarps * kMaxGroup * 2 * 4;
    static constexpr int kRedOff = kRingBytes;
    static constexpr int kBarOff = kRedOff + kRedOBytes + kRedMLBytes;
    // One barrier per stage and warp, plus one spare per warp (used only by
    // the wait-timeout test build, below).
    static constexpr int kBarBytes = (kWarps * (kStages + 1) * 8 + 127) / 128 * 128;
    static constexpr int kPrefixOff = kBarOff + kBarBytes;
    static constexpr int kSmemGrid = kPrefixOff;
    // Persistent grid: the chunk prefix, then (shared-prefix call) one bit
    // per sequence marking the grouped ones.
    static constexpr int kGroupedOff = kPrefixOff + (kMaxPersistSeqs + 1) * 4;
    static constexpr int kSmemPersist = kGroupedOff + (kMaxPersistSeqs + 31) / 32 * 4;
    static_assert(kRingBytes % 1024 == 0, "ring tiles must stay 1024-aligned");
    static_assert(kSmemPersist + 1024 <= 232448 / kTargetCtasPerSM,
                  "two CTAs per SM must fit");
};

// A piece of work: tokens [tok0, tok1) of sequence s for one kv head, and
// where its result goes.
enum PieceKind { kWhole = 0, kSlot = 1, kStraddle = 2 };

struct Item {
    int s;       // sequence; -1 = no item
    int L;       // context length (clamped)
    int tok0;    // first token
    int tok1;    // one past the last token
    int x1;      // persistent grid: chunk position one past the piece
    int kind;    // kWhole: the sequence's output; kSlot: partition idx's
                 // partial; kStraddle: the partial in this CTA's straddle row
    int idx;
};

__device__ __forceinline__ int clamped_len(const DecodeParams& p, int s) {
    int L = p.context_lens[s];
    if (L < 0 || L > p.max_context_len) {
        if ((threadIdx.x & 31) == 0) report(p.error_flags, PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : p.max_context_len;
    }
    return L;
}

__device__ __forceinline__ int parts_of(int L, int P) {
    return L <= 0 ? 1 : (L + P - 1) / P;  // an empty context still owns one item
}

// Sequence s has no items here: a shared-prefix group pass answers it (it
// belongs to a valid group with a prefix).
__device__ __forceinline__ bool grouped(const DecodeParams& p, int s) {
    const int i = cascade_group_of(p.groups, s);
    return i >= 0 && cascade_group_prefix(p.groups, i, p.num_seqs, p.block_size,
                                          nullptr, false) > 0;
}
template <bool kSkip>
__device__ __forceinline__ bool skipped(const DecodeParams& p, int s) {
    return kSkip && grouped(p, s);
}
// The same from the CTA's bitmap of grouped sequences (persistent grid).
template <bool kSkip>
__device__ __forceinline__ bool skipped_bit(const uint32_t* bits, int s) {
    return kSkip && ((bits[s >> 5] >> (s & 31)) & 1u);
}

// ---------------------------------------------------------------- plain grid
// One CTA per (kv head, partition, sequence); a partition past the
// sequence's end has no item.
__device__ __forceinline__ Item grid_item(const DecodeParams& p, int s, int part,
                                          bool skip) {
    Item it;
    it.s = -1;
    if (skip) return it;
    const int L = clamped_len(p, s);
    const int np = parts_of(L, p.partition_size);
    if (part >= np) return it;
    it.s = s;
    it.L = L;
    it.tok0 = part * p.partition_size;
    it.tok1 = min(L, it.tok0 + p.partition_size);
    it.x1 = 0;
    it.kind = np == 1 ? kWhole : kSlot;
    it.idx = part;
    return it;
}

// ---------------------------------------------------------- persistent grid
// Per kv head the 16-token chunks of all (not skipped) sequences lie end to
// end: sequence s occupies chunk positions [X[s], X[s+1]), T = X[B] in all.
// Split (max_partitions > 1): each warp of the head's CTAs is a range worker;
// worker i of the head's n takes positions [floor(i T/n), floor((i+1) T/n)),
// so every worker streams the same amount to within one chunk, and streams
// it alone: no warp of the CTA ever waits for another.  Its range is cut
// into pieces at sequence ends and at partition starts (every partition_size
// tokens of a sequence), so a partial never spans two partitions: a piece
// that starts a partition writes that partition's slot, the piece a worker
// starts in the middle of a partition writes the worker's straddle row, and
// a piece holding a whole sequence writes the output.  No split (the
// shared-prefix call's per-sequence pass): each CTA is one worker whose four
// warps share its items, and its range is the sequences whose first chunk
// lies in [floor(b T/n), floor((b+1) T/n)), taken whole.
struct Range {
    int r0, r1;   // chunk positions [r0, r1)
    int q;        // chunks per partition
    int worker;   // straddle row of a piece that starts mid-partition
};

// Largest s with X[s] <= x (x < X[B]): the sequence holding chunk x.
__device__ __forceinline__ int seq_at(const int* X, int B, int x) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (X[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Smallest sequence start X[s] >= x (X[B] if none).
__device__ __forceinline__ int seq_start_at_or_after(const int* X, int B, int x) {
    int lo = 0, hi = B;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (X[mid] >= x) hi = mid; else lo = mid + 1;
    }
    return X[lo];
}

__device__ __forceinline__ Item piece_at(const DecodeParams& p, const int* X,
                                         const Range& r, int x0) {
    Item it;
    it.s = -1;
    if (x0 >= r.r1) return it;
    const int s = seq_at(X, p.num_seqs, x0);
    const int xs = X[s];
    const int cs = X[s + 1] - xs;
    const int o0 = x0 - xs;
    const int k = o0 / r.q;
    const int pend = xs + min(cs, (k + 1) * r.q);
    it.s = s;
    it.L = clamped_len(p, s);
    it.x1 = min(pend, r.r1);
    it.tok0 = o0 * kChunk;
    it.tok1 = min(it.L, (it.x1 - xs) * kChunk);
    if (o0 == 0 && it.x1 == xs + cs) {
        it.kind = kWhole;
        it.idx = 0;
    } else if (o0 % r.q == 0) {
        it.kind = kSlot;
        it.idx = k;
    } else {
        it.kind = kStraddle;  // only a range's first piece starts mid-partition
        it.idx = r.worker;
    }
    return it;
}

// Chunks of `it` that warp w owns: all of them when the warp is a range
// worker, else chunks w, w+4, w+8, ... (the CTA's four warps share the item).
template <bool kWarpRanges>
__device__ __forceinline__ int warp_chunks(const Item& it, int warp) {
    if (it.s < 0) return 0;
    const int n = (it.tok1 - it.tok0 + kChunk - 1) / kChunk;
    if (kWarpRanges) return n;
    return n > warp ? (n - warp + kWarps - 1) / kWarps : 0;
}

// First token of the i-th chunk that warp w owns in `it`.
template <bool kWarpRanges>
__device__ __forceinline__ int chunk_token(const Item& it, int warp, int i) {
    return it.tok0 + (kWarpRanges ? i : warp + kWarps * i) * kChunk;
}

// Grid shapes of the partition kernel.
enum DecodeMode { kModeGrid = 0, kModeCtaRanges = 1, kModeWarpRanges = 2 };

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map,
                                            int c0, int c1, int c2,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::"
        "complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2),
        "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kThreads) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(int id) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(kThreads) : "memory");
}

template <int D, int BS, int kMode, bool kSkip>
__global__ void __launch_bounds__(kThreads, kTargetCtasPerSM)
paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const DecodeParams p) {
    using C = Cfg<D>;
    constexpr bool kPersist = kMode != kModeGrid;
    constexpr bool kWarpRanges = kMode == kModeWarpRanges;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char* ring = smem;
    float* red_o = reinterpret_cast<float*>(smem + C::kRedOff);
    float* red_m = red_o + (kWarps - 1) * kMaxGroup * C::kRedStride;
    float* red_l = red_m + kWarps * kMaxGroup;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    int* X = reinterpret_cast<int*>(smem + C::kPrefixOff);

    const int g = blockIdx.x;  // kv head
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.group;
    const int Hq = p.num_heads;

    // The 128-byte swizzle of the TMA tiles is tied to 1024-byte alignment.
    if (smem_u32(ring) & 1023u) {
        if (threadIdx.x == 0) report(p.error_flags, PA_DEVERR_INTERNAL);
        return;
    }
    // Launched behind the cache write: nothing global is read before the
    // preceding grid has completed.
    pdl_wait();
    pdl_launch_dependents();

    if (p.zero_count > 0) {
        // Each CTA clears a contiguous share.
        const long long ctas = (long long)gridDim.x * gridDim.y * gridDim.z;
        const long long me = ((long long)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
        const long long z0 = p.zero_count * me / ctas, z1 = p.zero_count * (me + 1) / ctas;
        for (long long z = z0 + threadIdx.x; z < z1; z += kThreads) p.zero_ints[z] = 0;
    }
    Range rg{0, 0, 1, 0};
    uint32_t* grouped_bits = reinterpret_cast<uint32_t*>(smem + C::kGroupedOff);
    if (kPersist && kSkip) {
        // Mark the members of every valid group with a prefix: a thread per
        // group, one round of loads (the same rule as cascade_group_prefix).
        for (int w = threadIdx.x; w < (p.num_seqs + 31) / 32; w += kThreads)
            grouped_bits[w] = 0u;
        __syncthreads();
        for (int i = threadIdx.x; i < p.groups.num_groups; i += kThreads) {
            if (cascade_group_prefix(p.groups, i, p.num_seqs, p.block_size, nullptr,
                                     false) <= 0)
                continue;
            const int a = p.groups.group_start[i], b = p.groups.group_start[i + 1];
            for (int s = a; s < b; ++s) atomicOr(&grouped_bits[s >> 5], 1u << (s & 31));
        }
        __syncthreads();
        if (!kWarpRanges) {
            // Every sequence answered by the group pass: nothing to stream
            // and no output to write (no merge follows without a split).
            bool any = false;
            for (int w = threadIdx.x; w < (p.num_seqs + 31) / 32; w += kThreads) {
                const uint32_t mine = w == (p.num_seqs - 1) / 32 && (p.num_seqs & 31)
                                          ? (1u << (p.num_seqs & 31)) - 1u
                                          : 0xffffffffu;
                any = any || (grouped_bits[w] & mine) != mine;
            }
            if (__syncthreads_or(any) == 0) return;
        }
    }
    if (kPersist) {
        // X[s] = 16-token chunks of sequences 0..s-1 (block-wide scan).  The
        // merge area is free until the first item ends; it holds the warp sums.
        int* warp_tot = reinterpret_cast<int*>(red_l);
        int running = 0;
        if (threadIdx.x == 0) X[0] = 0;
        for (int base = 0; base < p.num_seqs; base += kThreads) {
            const int s = base + threadIdx.x;
            int v = 0;
            if (s < p.num_seqs && !skipped_bit<kSkip>(grouped_bits, s))
                v = (clamped_len(p, s) + kChunk - 1) / kChunk;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += t;
            }
            if (lane == 31) warp_tot[warp] = v;
            __syncthreads();
            int before = running;
            for (int w = 0; w < warp; ++w) before += warp_tot[w];
            if (s < p.num_seqs) X[s + 1] = before + v;
            for (int w = 0; w < kWarps; ++w) running += warp_tot[w];
            __syncthreads();
        }
        const long long T = X[p.num_seqs];
        rg.q = p.partition_size / kChunk;
        if (kWarpRanges) {
            const long long n = (long long)gridDim.y * kWarps;
            rg.worker = blockIdx.y * kWarps + warp;
            rg.r0 = (int)(rg.worker * T / n);
            rg.r1 = (int)((rg.worker + 1) * T / n);
            // The merge kernel finds the pieces of a sequence from the same
            // scan and the same ranges.
            if (g == 0 && blockIdx.y == 0) {
                for (int s = threadIdx.x; s <= p.num_seqs; s += kThreads)
                    p.chunk_prefix[s] = X[s];
                for (int i = threadIdx.x; i <= n; i += kThreads)
                    p.worker_bounds[i] = (int)(i * T / n);
            }
            // Arrival counters of the merge, zeroed here: the merge kernel
            // starts only after this grid has completed.  Each CTA clears a
            // contiguous share.
            {
                const long long total = (long long)p.num_seqs * p.num_heads;
                const long long ctas = (long long)gridDim.x * gridDim.y;
                const long long me = (long long)blockIdx.y * gridDim.x + blockIdx.x;
                const long long c0 = total * me / ctas, c1 = total * (me + 1) / ctas;
                for (long long c = c0 + threadIdx.x; c < c1; c += kThreads) p.merge_count[c] = 0;
            }
        } else {
            const long long n = gridDim.y;
            const int b = blockIdx.y;
            rg.worker = b;
            rg.r0 = seq_start_at_or_after(X, p.num_seqs, (int)(b * T / n));
            rg.r1 = seq_start_at_or_after(X, p.num_seqs, (int)((b + 1) * T / n));
        }
    }
    // Items of this CTA, as a chain: key = chunk position of the piece's
    // start (persistent grid) or 0 / 1 = the CTA's one item / none (plain
    // grid).
    auto item_at = [&](int key) -> Item {
        if (kPersist) return piece_at(p, X, rg, key);
        Item none;
        none.s = -1;
        if (key != 0) return none;
        return grid_item(p, blockIdx.z, blockIdx.y, skipped<kSkip>(p, blockIdx.z));
    };
    auto next_key = [&](const Item& it) -> int { return kPersist ? it.x1 : 1; };
    const int first_key = kPersist ? rg.r0 : 0;

    uint64_t* my_bars = bars + warp * C::kStages;
    unsigned char* my_ring = ring + warp * C::kStages * C::kStageBytes;
    if (lane == 0) {
        for (int i = 0; i < C::kStages; ++i) mbar_init(&my_bars[i], 1);
#ifdef PA_TEST_UNSIGNALLED_FIRST_WAIT
        mbar_init(&bars[kWarps * C::kStages + warp], 1);
#endif
        mbar_init_fence();
    }
    __syncthreads();  // barriers initialised, prefix visible

    const int qr = lane >> 2;       // fragment row owned by this lane
    const int qc = (lane & 3) * 2;  // fragment column pair
    const int xr = lane & 7;        // swizzle phase of this lane's ldmatrix row
    const int mi = lane >> 3;       // ldmatrix sub-matrix this lane addresses

    const uint64_t pol = l2_policy_evict_first();
    const int32_t* tables = p.block_tables;
    const float sl2 = p.scale_log2;

    // ---------------- producer state (this warp's chunk stream) ----------
    int prod_key = first_key;  // item of the next chunk to look up
    int prod_i = 0;            // warp-chunk index within that item
    int prod_count = 0;        // chunks issued so far
    int ids_base = 0;          // prod_count at the last refill
    int ids = -1;              // lane l: slot coordinate of chunk ids_base + l
    bool prod_done = false;

    // Lane l finds the (ids_base + l)-th chunk of the stream and its slot.
    auto refill = [&]() {
        int key = prod_key, i = prod_i, n = lane;
        Item it = item_at(key);
        for (;;) {
            if (it.s < 0) break;
            const int rem = warp_chunks<kWarpRanges>(it, warp) - i;
            if (rem > n) break;
            n -= rem > 0 ? rem : 0;
            key = next_key(it);
            i = 0;
            it = item_at(key);
        }
        int slot = -1;
        if (it.s >= 0) {
            i += n;
            const int ctok = chunk_token<kWarpRanges>(it, warp, i);
            int id = tables[(int64_t)it.s * p.max_blocks_per_seq + ctok / BS];
            if (id < 0 || id >= p.num_blocks) {
                report(p.error_flags, PA_DEVERR_BLOCK_ID);
                id = 0;
            }
            slot = id * BS + ctok % BS;
            ++i;  // position after this lane's chunk
        }
        ids = slot;
        ids_base = prod_count;
        prod_key = __shfl_sync(0xffffffffu, key, 31);
        prod_i = __shfl_sync(0xffffffffu, i, 31);
        prod_done = __shfl_sync(0xffffffffu, slot, 31) < 0;
    };

    // Issue the next chunk of the stream into its stage; false when none.
    auto issue = [&]() -> bool {
        if (prod_count == ids_base + 32 || prod_count == 0) {
            if (prod_count == 0 || !prod_done) refill();
        }
        const int slot = __shfl_sync(0xffffffffu, ids, (prod_count - ids_base) & 31);
        if (slot < 0 || prod_count - ids_base >= 32) return false;
        const int stage = prod_count % C::kStages;
        const uint32_t dst = smem_u32(my_ring + stage * C::kStageBytes);
        uint64_t* bar = &my_bars[stage];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive_expect_tx(bar, C::kStageBytes);
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h) {
                tma_load_3d(dst + h * C::kHalfBytes, &tm_k, 0, g * C::kHalves + h,
                            slot, bar, pol);
                tma_load_3d(dst + C::kKVBytes + h * C::kHalfBytes, &tm_v, 0,
                            g * C::kHalves + h, slot, bar, pol);
            }
        }
        ++prod_count;
        return true;
    };

    for (int j = 0; j < C::kStages; ++j)
        if (!issue()) break;

    // ---------------- consumer ----------------
    int cons_count = 0;
    bool aborted = false;
    int drain_from = 0;  // first chunk whose wait gave up
    int items_done = 0;
    // Q fragments of an item (A operand): rows = heads of the group, rows >= G
    // zero.  The next item's are fetched while the current one streams.
    auto load_q = [&](const Item& it, uint32_t (&dst)[D / 16][2]) {
        const bool live = it.s >= 0 && qr < G && it.L > 0;
        const uint16_t* qp =
            p.q + ((int64_t)(it.s < 0 ? 0 : it.s) * Hq + g * G + (qr < G ? qr : 0)) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            dst[ks][0] = live ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + qc) : 0u;
            dst[ks][1] = live ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8 + qc) : 0u;
        }
    };
    Item next_it = item_at(first_key);
    uint32_t qnext[D / 16][2];
    load_q(next_it, qnext);
    for (;;) {
        const Item it = next_it;
        if (it.s < 0) break;
        const int my_n = warp_chunks<kWarpRanges>(it, warp);
        uint32_t qa[D / 16][2];
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = qnext[ks][0];
            qa[ks][1] = qnext[ks][1];
        }
        next_it = item_at(next_key(it));
        load_q(next_it, qnext);

        float o[D / 8][4];
#pragma unroll
        for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        float m_run = -INFINITY;
        float l_run = 0.f;

        for (int i = 0; i < my_n; ++i) {
            const int stage = cons_count % C::kStages;
            if (!aborted) {
#ifdef PA_TEST_UNSIGNALLED_FIRST_WAIT
                const bool ok =
                    cons_count == 0
                        ? mbar_wait_bounded(&bars[kWarps * C::kStages + warp], 0,
                                            kTestWaitLimitNs)
                        : mbar_wait_bounded(&my_bars[stage], (cons_count / C::kStages) & 1);
#else
                const bool ok = mbar_wait_bounded(&my_bars[stage],
                                                  (cons_count / C::kStages) & 1);
#endif
                if (!__all_sync(0xffffffffu, ok)) {
                    aborted = true;
                    drain_from = cons_count;
                    if (lane == 0) report(p.error_flags, PA_DEVERR_TIMEOUT);
                }
            }
            ++cons_count;
            if (aborted) continue;

            const int ctok = chunk_token<kWarpRanges>(it, warp, i);
            const int valid = min(kChunk, it.tok1 - ctok);
            const uint32_t kaddr = smem_u32(my_ring + stage * C::kStageBytes);
            const uint32_t vaddr = kaddr + C::kKVBytes;

            if (valid < kChunk) {
                // Rows past the context hold whatever the block holds; V must
                // be finite there because P is zero.
                const int rows = kChunk - valid;
                for (int e = lane; e < rows * C::kHalves * 8; e += 32) {
                    const int r = valid + e / (C::kHalves * 8);
                    const int h = (e / 8) % C::kHalves;
                    const int c = e & 7;
                    const uint32_t a = vaddr + h * C::kHalfBytes + r * 128 + c * 16;
                    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(a), "r"(0)
                                 : "memory");
                }
                __syncwarp();
            }

            // S (16 rows x 16 tokens) = Q K^T: two n8 tiles, two k chains each.
            float sacc[2][2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
                    sacc[nt][ch][0] = sacc[nt][ch][1] = sacc[nt][ch][2] = sacc[nt][ch][3] = 0.f;
                const uint32_t row = kaddr + (nt * 8 + xr) * 128;
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk) {
                    const int cidx = ((kk & 1) << 2) + mi;
                    const uint32_t a = row + (kk >> 1) * C::kHalfBytes + ((cidx ^ xr) << 4);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(b0, b1, b2, b3, a);
                    mma_bf16_16816(sacc[nt][kk & 1], qa[2 * kk][0], 0u, qa[2 * kk][1], 0u, b0, b1);
                    mma_bf16_16816(sacc[nt][kk & 1], qa[2 * kk + 1][0], 0u, qa[2 * kk + 1][1], 0u, b2, b3);
                }
            }

            float sv[4];
            if (valid == kChunk) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        sv[nt * 2 + e] = (sacc[nt][0][e] + sacc[nt][1][e]) * sl2;
            } else {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        sv[nt * 2 + e] = (nt * 8 + qc + e < valid)
                                             ? (sacc[nt][0][e] + sacc[nt][1][e]) * sl2
                                             : -INFINITY;
            }
            float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            if (__any_sync(0xffffffffu, mx > m_run)) {
                const float m_new = fmaxf(m_run, mx);
                const float alpha = exp2f(m_run - m_new);
                m_run = m_new;
                l_run *= alpha;
#pragma unroll
                for (int j2 = 0; j2 < D / 8; ++j2) {
                    o[j2][0] *= alpha; o[j2][1] *= alpha;
                    o[j2][2] *= alpha; o[j2][3] *= alpha;
                }
            }
            float pv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) pv[e] = exp2f(sv[e] - m_run);
            l_run += (pv[0] + pv[1]) + (pv[2] + pv[3]);

            // P as the A operand: rows 0..7 = bf16(P), rows 8..15 = bf16(P - bf16(P)).
            const float h0 = bf16_round(pv[0]), h1 = bf16_round(pv[1]);
            const float h2 = bf16_round(pv[2]), h3 = bf16_round(pv[3]);
            const uint32_t a0 = pack_bf16x2(h0, h1);
            const uint32_t a2 = pack_bf16x2(h2, h3);
            const uint32_t a1 = pack_bf16x2(pv[0] - h0, pv[1] - h1);
            const uint32_t a3 = pack_bf16x2(pv[2] - h2, pv[3] - h3);

            // O (16 x D) += P (16 x 16 tokens) V (16 tokens x D).
            const uint32_t vrow = vaddr + (((mi & 1) << 3) + xr) * 128;
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                const int cidx = ((dp & 3) << 1) + (mi >> 1);
                const uint32_t a = vrow + (dp >> 2) * C::kHalfBytes + ((cidx ^ xr) << 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_trans(b0, b1, b2, b3, a);
                mma_bf16_16816(o[2 * dp], a0, a1, a2, a3, b0, b1);
                mma_bf16_16816(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
            }
            __syncwarp();
            if (!prod_done || prod_count < ids_base + 32) issue();
        }

        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
        if (kWarpRanges) {
            // ------------- item end of a range worker: its own result ---
            // Rows qr (the head) and qr + 8 (the P residual's share) add up;
            // the quad's lanes hold the row's columns 8j + qc, +1.
            if (qr < G) {
                const int h = g * G + qr;
                const int64_t row = (int64_t)it.s * Hq + h;
                int64_t pidx = 0;
                float* dst;
                if (it.kind == kWhole) {
                    dst = p.out + row * D;
                } else if (it.kind == kSlot) {
                    pidx = row * p.max_partitions + it.idx;
                    dst = p.tmp_o + pidx * D;
                } else {
                    pidx = (int64_t)h * p.max_range_workers + it.idx;
                    dst = p.st_o + pidx * D;
                }
                const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
                if (it.kind == kWhole) {
#pragma unroll
                    for (int j = 0; j < D / 8; ++j)
                        *reinterpret_cast<float2*>(dst + 8 * j + qc) =
                            make_float2((o[j][0] + o[j][2]) * inv, (o[j][1] + o[j][3]) * inv);
                } else {
                    // A partial: kept in L2 for the merge kernel, which reads
                    // it right after this grid while the KV stream evicts.
                    const uint64_t keep = l2_policy_evict_last();
#pragma unroll
                    for (int j = 0; j < D / 8; ++j)
                        st_global_f2_hint(dst + 8 * j + qc, (o[j][0] + o[j][2]) * inv,
                                          (o[j][1] + o[j][3]) * inv, keep);
                }
                if (it.kind != kWhole && (lane & 3) == 0) {
                    float* dm = it.kind == kSlot ? p.tmp_m : p.st_m;
                    float* dl = it.kind == kSlot ? p.tmp_l : p.st_l;
                    dm[pidx] = m_run;
                    dl[pidx] = l_run;
                }
            }
            continue;
        }
        // ---------------- item end: merge the four warps ----------------
        // Warps 1..3 post (max, sum, O) and go on streaming; warp 0 merges
        // and writes the result, so only warp 0 pauses its copy ring.
        if (warp != 0) {
            if (items_done > 0) named_bar_sync(2);  // warp 0 has read the previous item
            float* dst = red_o + ((warp - 1) * kMaxGroup + qr) * C::kRedStride + qc;
#pragma unroll
            for (int j = 0; j < D / 8; ++j)
                *reinterpret_cast<float2*>(dst + 8 * j) =
                    make_float2(o[j][0] + o[j][2], o[j][1] + o[j][3]);
            if ((lane & 3) == 0) {
                red_m[warp * kMaxGroup + qr] = m_run;
                red_l[warp * kMaxGroup + qr] = l_run;
            }
            named_bar_arrive(1);
        } else {
            named_bar_sync(1);
            float sc[kWarps], M = m_run;
#pragma unroll
            for (int w = 1; w < kWarps; ++w) M = fmaxf(M, red_m[w * kMaxGroup + qr]);
            float den = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float mw = w == 0 ? m_run : red_m[w * kMaxGroup + qr];
                const float lw = w == 0 ? l_run : red_l[w * kMaxGroup + qr];
                sc[w] = mw == -INFINITY ? 0.f : exp2f(mw - M);
                den += sc[w] * lw;
            }
            if (qr < G) {
                const int h = g * G + qr;
                const int64_t row = (int64_t)it.s * Hq + h;
                int64_t pidx = 0;
                float* dst;
                if (it.kind == kWhole) {
                    dst = p.out + row * D;
                } else if (it.kind == kSlot) {
                    pidx = row * p.max_partitions + it.idx;
                    dst = p.tmp_o + pidx * D;
                } else {
                    pidx = (int64_t)h * p.max_range_workers + it.idx;
                    dst = p.st_o + pidx * D;
                }
#pragma unroll
                for (int j = 0; j < D / 8; ++j) {
                    float v[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float acc = sc[0] * (o[j][e] + o[j][e + 2]);
#pragma unroll
                        for (int w = 1; w < kWarps; ++w)
                            acc += sc[w] * red_o[((w - 1) * kMaxGroup + qr) * C::kRedStride + 8 * j + qc + e];
                        v[e] = it.L > 0 ? acc / den : 0.f;
                    }
                    *reinterpret_cast<float2*>(dst + 8 * j + qc) = make_float2(v[0], v[1]);
                }
                if (it.kind != kWhole && (lane & 3) == 0) {
                    float* dm = it.kind == kSlot ? p.tmp_m : p.st_m;
                    float* dl = it.kind == kSlot ? p.tmp_l : p.st_l;
                    dm[pidx] = M;
                    dl[pidx] = den;
                }
            }
            named_bar_arrive(2);
        }
        ++items_done;
    }
    // Consume warp 0's last "merged" arrival so no barrier is left pending.
    if (warp != 0 && items_done > 0) named_bar_sync(2);

    if (kPersist) {
        // Sequences with an empty context (not skipped) own no chunk: their
        // output is zero, written by the CTAs of the head in turn.
        for (int s = blockIdx.y; s < p.num_seqs; s += gridDim.y) {
            if (skipped_bit<kSkip>(grouped_bits, s) || X[s + 1] != X[s]) continue;
            for (int e = threadIdx.x; e < G * D; e += kThreads)
                p.out[((int64_t)s * Hq + g * G) * D + e] = 0.f;
        }
    }

    if (aborted) {
        // Drain copies still in flight on this warp's ring (bounded) before
        // the CTA exits.
        for (int c = drain_from; c < prod_count; ++c)
            (void)mbar_wait_bounded(&my_bars[c % C::kStages], (c / C::kStages) & 1);
    }
}

// ---------------------------------------------------------------- merges
// Merge of a split sequence's pieces: out = sum_i w_i o_i / sum_i w_i with
// w_i = l_i * 2^(m_i - max_j m_j).  A row of (m, l, o) of D floats per piece;
// rows are read 8 per warp per round, all loads of a round issued before any
// value is used, with a running max so a round is one memory round trip.
constexpr int kReduceWarps = 8;
constexpr int kReduceUnroll = 8;
static_assert(kReduceWarps * kReduceUnroll == kMergeRows, "one round per merge slice");

template <int D>
struct MergeAcc {
    static constexpr int V = D / 32;  // columns per lane
    float M = -INFINITY, den = 0.f;
    float acc[V] = {};

    // Fold a round of up to kReduceUnroll rows (live[u] false: ignored).
    __device__ __forceinline__ void fold(const float (&mv)[kReduceUnroll],
                                         const float (&lv)[kReduceUnroll],
                                         const float (&vals)[kReduceUnroll][V],
                                         const bool (&live)[kReduceUnroll]) {
        float Mr = M;
#pragma unroll
        for (int u = 0; u < kReduceUnroll; ++u)
            if (live[u]) Mr = fmaxf(Mr, mv[u]);
        if (Mr == -INFINITY) return;
        const float keep = M == -INFINITY ? 0.f : exp2f(M - Mr);
        den *= keep;
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] *= keep;
#pragma unroll
        for (int u = 0; u < kReduceUnroll; ++u) {
            if (!live[u] || mv[u] == -INFINITY) continue;
            const float w = lv[u] * exp2f(mv[u] - Mr);
            den += w;
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] += w * vals[u][v];
        }
        M = Mr;
    }
};

template <int D>
__device__ __forceinline__ void load_row(const float* row, bool ok, float (&dst)[D / 32]) {
    constexpr int V = D / 32;
    if (V == 4) {
        const float4 t = ok ? *reinterpret_cast<const float4*>(row) : make_float4(0.f, 0.f, 0.f, 0.f);
        dst[0] = t.x; dst[V > 1 ? 1 : 0] = t.y; dst[V > 2 ? 2 : 0] = t.z; dst[V > 3 ? 3 : 0] = t.w;
    } else {
        const float2 t = ok ? *reinterpret_cast<const float2*>(row) : make_float2(0.f, 0.f);
        dst[0] = t.x; dst[V > 1 ? 1 : 0] = t.y;
    }
}

// Combine the 8 warps' accumulators through shared memory; every thread
// returns the CTA's max and sum, and thread d's column d of the sum of O.
template <int D>
struct MergeSmem {
    float m[kReduceWarps];
    float den[kReduceWarps];
    float acc[kReduceWarps][D];
};

template <int D>
__device__ __forceinline__ void combine_warps(const MergeAcc<D>& a, MergeSmem<D>& sm,
                                              float& M, float& den) {
    constexpr int V = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        sm.m[warp] = a.M;
        sm.den[warp] = a.den;
    }
#pragma unroll
    for (int v = 0; v < V; ++v) sm.acc[warp][lane * V + v] = a.acc[v];
    __syncthreads();
    M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w) M = fmaxf(M, sm.m[w]);
    den = 0.f;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w)
        den += sm.m[w] == -INFINITY ? 0.f : sm.den[w] * exp2f(sm.m[w] - M);
}

template <int D>
__device__ __forceinline__ float combined_column(const MergeSmem<D>& sm, float M, int d) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w)
        a += sm.m[w] == -INFINITY ? 0.f : sm.acc[w][d] * exp2f(sm.m[w] - M);
    return a;
}

// Plain grid (more than kMaxPersistSeqs sequences): one CTA of 8 warps per
// (query head, sequence) merges the sequence's partition slots.  Sequences
// held by one partition were written by the partition kernel.
template <int D>
__global__ void __launch_bounds__(kReduceWarps * 32, 3)
paged_decode_reduce_kernel(const DecodeParams p) {
    constexpr int V = D / 32;
    const int h = blockIdx.x;
    const int s = blockIdx.y;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    pdl_wait();  // the partials come from the grid launched just before
    int L = p.context_lens[s];
    if (p.has_groups && grouped(p, s)) return;  // answered by the group pass
    L = L < 0 ? 0 : (L > p.max_context_len ? p.max_context_len : L);
    const int nslot = (L + p.partition_size - 1) / p.partition_size;
    if (nslot <= 1) return;
    __shared__ MergeSmem<D> sm;
    const int64_t base = ((int64_t)s * p.num_heads + h) * p.max_partitions;
    MergeAcc<D> a;
    for (int i0 = warp; i0 < nslot; i0 += kReduceWarps * kReduceUnroll) {
        float mv[kReduceUnroll], lv[kReduceUnroll], vals[kReduceUnroll][V];
        bool live[kReduceUnroll];
#pragma unroll
        for (int u = 0; u < kReduceUnroll; ++u) {
            const int i = i0 + u * kReduceWarps;
            live[u] = i < nslot;
            const int64_t r = base + (live[u] ? i : 0);
            mv[u] = live[u] ? p.tmp_m[r] : -INFINITY;
            lv[u] = live[u] ? p.tmp_l[r] : 0.f;
            load_row<D>(p.tmp_o + r * D + lane * V, live[u], vals[u]);
        }
        a.fold(mv, lv, vals, live);
    }
    float M, den;
    combine_warps<D>(a, sm, M, den);
    for (int d = threadIdx.x; d < D; d += kReduceWarps * 32)
        p.out[((int64_t)s * p.num_heads + h) * D + d] = combined_column<D>(sm, M, d) / den;
}

// Candidate rows of a split sequence for one query head: its partition
// slots, then the range boundaries strictly inside it (live when the
// boundary is no partition start and is the last worker starting there).
// Loads rows i0 + u * step (u < kReduceUnroll, those below total) in one
// round and folds them into a.
template <int D>
__device__ __forceinline__ void fold_candidates(const DecodeParams& p, MergeAcc<D>& a, int i0,
                                                int step, int total, int nslot, int b_lo, int xs,
                                                int q, int nw, int64_t slot_base,
                                                int64_t st_base, int lane) {
    constexpr int V = D / 32;
    const int32_t* E = p.worker_bounds;
    float mv[kReduceUnroll], lv[kReduceUnroll], vals[kReduceUnroll][V];
    int e0[kReduceUnroll], e1[kReduceUnroll];
    bool live[kReduceUnroll], in_slots[kReduceUnroll];
#pragma unroll
    for (int u = 0; u < kReduceUnroll; ++u) {
        const int i = i0 + u * step;
        const bool ok = i < total;
        in_slots[u] = i < nslot;
        const int b = min(max(b_lo + i - nslot, 0), nw - 1);
        const int64_t r = in_slots[u] ? slot_base + i : st_base + b;
        e0[u] = (ok && !in_slots[u]) ? E[b] : 0;
        e1[u] = (ok && !in_slots[u]) ? E[b + 1] : 0;
        mv[u] = ok ? (in_slots[u] ? p.tmp_m : p.st_m)[r] : -INFINITY;
        lv[u] = ok ? (in_slots[u] ? p.tmp_l : p.st_l)[r] : 0.f;
        load_row<D>((in_slots[u] ? p.tmp_o : p.st_o) + r * D + lane * V, ok, vals[u]);
        live[u] = ok;
    }
#pragma unroll
    for (int u = 0; u < kReduceUnroll; ++u)
        live[u] = live[u] && (in_slots[u] || ((e0[u] - xs) % q != 0 && e1[u] > e0[u]));
    a.fold(mv, lv, vals, live);
}

// A split sequence with at most this many candidate rows is merged by one
// warp; longer ones by CTAs, kMergeRows rows per slice.
constexpr int kWarpMergeMax = 2 * kReduceUnroll;

// Range-worker grid: a persistent grid over the split sequences.  Each CTA
// scans the published chunk prefix into two work lists.  Long sequences
// (more than kWarpMergeMax candidate rows) are merged by CTA items
// (sequence, query head, slice of kMergeRows rows), one round per slice: a
// sequence with one slice is written at once, otherwise each slice writes
// its (max, sum, normalised O) and the last of the sequence's slices to
// arrive (an arrival counter the partition kernel zeroed) merges them.
// Short ones (most split sequences: two or three pieces) are merged whole by
// one warp per (sequence, query head), in one or two rounds with no CTA
// barrier.  A CTA takes its long items first, so the slices that gate a
// second level are done early.  No CTA waits on another.
template <int D>
__global__ void __launch_bounds__(kReduceWarps * 32, 2)
paged_decode_merge_kernel(const DecodeParams p) {
    constexpr int V = D / 32;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int Hq = p.num_heads;
    // Per sequence, computed once by the CTA: CTA slices and warp items (as
    // prefixes over sequences: the work lists), partition slots, first
    // boundary candidate, candidate count and first chunk.
    __shared__ int work[kMaxPersistSeqs + 1], work_w[kMaxPersistSeqs + 1];
    __shared__ int g_nslot[kMaxPersistSeqs], g_blo[kMaxPersistSeqs];
    __shared__ int g_total[kMaxPersistSeqs], g_xs[kMaxPersistSeqs];
    __shared__ int wsum[2][kReduceWarps];
    __shared__ MergeSmem<D> sm;
    __shared__ int is_last;
    pdl_wait();  // the partials come from the grid launched just before

    const long long T = p.chunk_prefix[p.num_seqs];
    const int nw = p.range_workers;
    const int q = p.partition_size / kChunk;
    int running = 0, running_w = 0;
    if (threadIdx.x == 0) {
        work[0] = 0;
        work_w[0] = 0;
    }
    for (int base = 0; base < p.num_seqs; base += kReduceWarps * 32) {
        const int s = base + threadIdx.x;
        int v = 0, vw = 0;
        if (s < p.num_seqs) {
            const long long xs = p.chunk_prefix[s];
            const long long cs = p.chunk_prefix[s + 1] - xs;
            int nslot = 0, b_lo = 1, ncand = 0;
            if (cs > 0) {
                nslot = (int)((cs + q - 1) / q);
                const long long lo = max(1LL, ((xs + 1) * nw + T - 1) / T);
                const long long hi = min((long long)nw - 1, ((xs + cs) * nw + T - 1) / T - 1);
                b_lo = (int)lo;
                ncand = hi >= lo ? (int)(hi - lo + 1) : 0;
                // Two slots, or one slot and a boundary inside: split.
                if (nslot >= 2 || ncand >= 1) {
                    if (nslot + ncand <= kWarpMergeMax) vw = 1;
                    else v = (nslot + ncand + kMergeRows - 1) / kMergeRows;
                }
            }
            g_nslot[s] = nslot;
            g_blo[s] = b_lo;
            g_total[s] = nslot + ncand;
            g_xs[s] = (int)xs;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, v, o);
            const int tw = __shfl_up_sync(0xffffffffu, vw, o);
            if (lane >= o) {
                v += t;
                vw += tw;
            }
        }
        if (lane == 31) {
            wsum[0][warp] = v;
            wsum[1][warp] = vw;
        }
        __syncthreads();
        int before = running, before_w = running_w;
        for (int w = 0; w < warp; ++w) {
            before += wsum[0][w];
            before_w += wsum[1][w];
        }
        if (s < p.num_seqs) {
            work[s + 1] = before + v;
            work_w[s + 1] = before_w + vw;
        }
        for (int w = 0; w < kReduceWarps; ++w) {
            running += wsum[0][w];
            running_w += wsum[1][w];
        }
        __syncthreads();
    }
    const int total_items = running * Hq;
    // Largest s with list[s] <= k.
    auto seq_of = [&](const int* list, int k) {
        int lo = 0, hi = p.num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (list[mid] <= k) lo = mid; else hi = mid - 1;
        }
        return lo;
    };

    for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
        const int h = item % Hq;
        const int gsl = item / Hq;
        const int s = seq_of(work, gsl);
        const int sl = gsl - work[s];
        const int nsl = work[s + 1] - work[s];
        const int64_t slot_base = ((int64_t)s * Hq + h) * p.max_partitions;
        const int64_t st_base = (int64_t)h * p.max_range_workers;

        // First level: candidate rows [sl * kMergeRows, +kMergeRows), one round.
        MergeAcc<D> a;
        fold_candidates<D>(p, a, sl * kMergeRows + warp, kReduceWarps, g_total[s], g_nslot[s],
                           g_blo[s], g_xs[s], q, nw, slot_base, st_base, lane);
        float M, den;
        combine_warps<D>(a, sm, M, den);
        float* out_row = p.out + ((int64_t)s * Hq + h) * D;
        if (nsl == 1) {
            for (int d = threadIdx.x; d < D; d += kReduceWarps * 32)
                out_row[d] = combined_column<D>(sm, M, d) / den;
            __syncthreads();  // sm is reused by the next item
            continue;
        }
        const int64_t sub = ((int64_t)s * Hq + h) * p.max_slices;
        for (int d = threadIdx.x; d < D; d += kReduceWarps * 32)
            p.sub_o[(sub + sl) * D + d] =
                den > 0.f ? combined_column<D>(sm, M, d) / den : 0.f;
        if (threadIdx.x == 0) {
            p.sub_m[sub + sl] = den > 0.f ? M : -INFINITY;
            p.sub_l[sub + sl] = den;
        }
        // Publish the slice, then count it; the last slice to arrive merges.
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0)
            is_last = atomicAdd(&p.merge_count[(int64_t)s * Hq + h], 1) == nsl - 1;
        __syncthreads();
        if (!is_last) continue;
        __threadfence();
        MergeAcc<D> b;
        for (int i0 = warp; i0 < nsl; i0 += kReduceWarps * kReduceUnroll) {
            float mv[kReduceUnroll], lv[kReduceUnroll], vals[kReduceUnroll][V];
            bool live[kReduceUnroll];
#pragma unroll
            for (int u = 0; u < kReduceUnroll; ++u) {
                const int i = i0 + u * kReduceWarps;
                live[u] = i < nsl;
                const int64_t r = sub + (live[u] ? i : 0);
                // Written by other CTAs of this grid: read through L2.
                mv[u] = live[u] ? __ldcg(p.sub_m + r) : -INFINITY;
                lv[u] = live[u] ? __ldcg(p.sub_l + r) : 0.f;
                const float* row = p.sub_o + r * D + lane * V;
#pragma unroll
                for (int v = 0; v < V; ++v) vals[u][v] = live[u] ? __ldcg(row + v) : 0.f;
            }
            b.fold(mv, lv, vals, live);
        }
        combine_warps<D>(b, sm, M, den);
        for (int d = threadIdx.x; d < D; d += kReduceWarps * 32)
            out_row[d] = combined_column<D>(sm, M, d) / den;
        __syncthreads();
    }

    // Short split sequences: one warp per (sequence, query head), no barrier.
    const int total_w = running_w * Hq;
    for (int it = blockIdx.x * kReduceWarps + warp; it < total_w;
         it += gridDim.x * kReduceWarps) {
        const int h = it % Hq;
        const int s = seq_of(work_w, it / Hq);
        const int total = g_total[s];
        const int64_t slot_base = ((int64_t)s * Hq + h) * p.max_partitions;
        const int64_t st_base = (int64_t)h * p.max_range_workers;
        MergeAcc<D> a;
        for (int i0 = 0; i0 < total; i0 += kReduceUnroll)
            fold_candidates<D>(p, a, i0, 1, total, g_nslot[s], g_blo[s], g_xs[s], q, nw,
                               slot_base, st_base, lane);
        float* out_row = p.out + ((int64_t)s * Hq + h) * D + lane * V;
        const float inv = a.den > 0.f ? 1.f / a.den : 0.f;
#pragma unroll
        for (int v = 0; v < V; ++v) out_row[v] = a.acc[v] * inv;
    }
}

// ------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                   void*, const cuuint64_t*, const cuuint64_t*,
                                   const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr,
                                    cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// Pool [NB*bs][Hkv][D] viewed as 3-D {64 elements, Hkv*D/64 column tiles,
// NB*bs token slots}; box = one 128-byte column tile of 16 slots.
bool encode_pool_map(CUtensorMap* map, const void* pool, int num_blocks,
                     int block_size, int num_kv_heads, int head_size) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)num_kv_heads * head_size / 64,
                                (cuuint64_t)num_blocks * block_size};
    const cuuint64_t strides[2] = {128, (cuuint64_t)num_kv_heads * head_size * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kChunk};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch with a programmatic edge to the previous kernel in the stream: this
// grid may be scheduled while that one finishes and waits for it in-kernel.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block,
                       size_t smem, cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename Kernel>
cudaError_t set_smem(Kernel kernel, int bytes, int* flags) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!__atomic_load_n(&flags[dev], __ATOMIC_ACQUIRE)) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        __atomic_store_n(&flags[dev], 1, __ATOMIC_RELEASE);
    }
    return cudaSuccess;
}

template <int D, int BS, int kMode, bool kSkip>
cudaError_t launch_mode(const DecodeParams& p, const CUtensorMap& tmk,
                        const CUtensorMap& tmv, dim3 grid, int smem,
                        cudaStream_t stream) {
    static int ready[64] = {0};
    cudaError_t e = set_smem(paged_decode_kernel<D, BS, kMode, kSkip>, smem, ready);
    if (e != cudaSuccess) return e;
    e = launch_pdl(paged_decode_kernel<D, BS, kMode, kSkip>, grid, dim3(kThreads),
                   smem, stream, tmk, tmv, p);
    count_launch();
    return e;
}

// Persistent CTAs when sequences are split (balanced chunk ranges per warp),
// and when some sequences are skipped (no CTA is spent on them); up to
// kMaxPersistSeqs sequences, whose chunk prefix fits in shared memory.
template <int D, int BS, bool kSkip>
cudaError_t launch_partition_kernel(DecodeParams& p, const CUtensorMap& tmk,
                                    const CUtensorMap& tmv, cudaStream_t stream) {
    using C = Cfg<D>;
    p.range_workers = 0;
    const bool split = p.max_partitions > 1;
    if ((split || kSkip) && p.num_seqs <= kMaxPersistSeqs) {
        long long per_head = decode_ctas_per_head(p.num_kv_heads);
        const long long items = (long long)p.num_seqs * p.max_partitions;
        if (per_head > items) per_head = items;
        if (split && per_head * kWarps > p.max_range_workers)
            per_head = p.max_range_workers / kWarps;  // the straddle region's rows
        if (per_head < 1) per_head = 1;
        const dim3 grid((unsigned)p.num_kv_heads, (unsigned)per_head, 1);
        if (split) {
            p.range_workers = (int)per_head * kWarps;
            return launch_mode<D, BS, kModeWarpRanges, kSkip>(p, tmk, tmv, grid,
                                                             C::kSmemPersist, stream);
        }
        return launch_mode<D, BS, kModeCtaRanges, kSkip>(p, tmk, tmv, grid,
                                                        C::kSmemPersist, stream);
    }
    const dim3 grid((unsigned)p.num_kv_heads, (unsigned)p.max_partitions,
                    (unsigned)p.num_seqs);
    return launch_mode<D, BS, kModeGrid, kSkip>(p, tmk, tmv, grid, C::kSmemGrid, stream);
}

template <int D, int BS>
cudaError_t launch_typed(const DecodeParams& params, cudaStream_t stream) {
    CUtensorMap tmk, tmv;
    if (!encode_pool_map(&tmk, params.k_cache, params.num_blocks, BS, params.num_kv_heads, D) ||
        !encode_pool_map(&tmv, params.v_cache, params.num_blocks, BS, params.num_kv_heads, D))
        return cudaErrorInvalidValue;
    DecodeParams p = params;
    cudaError_t e = p.has_groups
                        ? launch_partition_kernel<D, BS, true>(p, tmk, tmv, stream)
                        : launch_partition_kernel<D, BS, false>(p, tmk, tmv, stream);
    if (e != cudaSuccess) return e;
    if (p.max_partitions > 1) {
        if (p.range_workers > 0) {
            // Persistent over the work list the partition kernel published.
            const dim3 mgrid((unsigned)(2 * device_sm_count()));
            e = launch_pdl(paged_decode_merge_kernel<D>, mgrid, dim3(kReduceWarps * 32), 0,
                           stream, p);
        } else {
            const dim3 rgrid((unsigned)p.num_heads, (unsigned)p.num_seqs);
            e = launch_pdl(paged_decode_reduce_kernel<D>, rgrid, dim3(kReduceWarps * 32), 0,
                           stream, p);
        }
        count_launch();
    }
    return e;
}

}  // namespace

float log2e_scale(float scale) { return scale * kLog2e; }

int decode_ctas_per_head(int num_kv_heads) {
    if (num_kv_heads <= 0) return 1;
    return (kTargetCtasPerSM * device_sm_count() + num_kv_heads - 1) / num_kv_heads;
}

int decode_range_workers(int num_kv_heads) {
    return kWarps * decode_ctas_per_head(num_kv_heads);
}

cudaError_t launch_paged_decode(const DecodeParams& p, int head_size,
                                int block_size, cudaStream_t stream) {
    if (head_size == 128 && block_size == 16) return launch_typed<128, 16>(p, stream);
    if (head_size == 128 && block_size == 32) return launch_typed<128, 32>(p, stream);
    if (head_size == 64 && block_size == 16) return launch_typed<64, 16>(p, stream);
    if (head_size == 64 && block_size == 32) return launch_typed<64, 32>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
