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
constexpr int kNumSMs = 148;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
    static constexpr int kHalves = D / 64;                  // 128-byte column tiles
    static constexpr int kHalfBytes = kChunk * 128;         // 16 rows x 128 B
    static constexpr int kKVBytes = kHalves * kHalfBytes;   // K (or V) of a chunk
    static constexpr int kStageBytes = 2 * kKVBytes;
    static constexpr int kStages = D == 128 ? 3 : 5;
    static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
    static constexpr int kRedStride = D + 8;                // floats per row
    static constexpr int kRedOBytes = (kWarps - 1) * kMaxGroup * kRedStride * 4;
    static constexpr int kRedMLBytes = kWarps * kMaxGroup * 2 * 4;
    static constexpr int kRedOff = kRingBytes;
    static constexpr int kBarOff = kRedOff + kRedOBytes + kRedMLBytes;
    static constexpr int kBarBytes = (kWarps * kStages * 8 + 127) / 128 * 128;
    static constexpr int kPrefixOff = kBarOff + kBarBytes;
    static constexpr int kSmemGrid = kPrefixOff;
    static constexpr int kSmemPersist = kPrefixOff + (kMaxPersistSeqs + 1) * 4;
    static_assert(kRingBytes % 1024 == 0, "ring tiles must stay 1024-aligned");
    static_assert(kSmemPersist + 1024 <= 232448 / kTargetCtasPerSM,
                  "two CTAs per SM must fit");
};

struct Item {
    int s;       // sequence; -1 = no item
    int part;    // partition index
    int L;       // context length (clamped)
    int tok0;    // first token of the partition
    int tok1;    // one past its last token
    int nparts;  // partitions of this sequence
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

// Sequence s has no items here: a shared-prefix group pass answered it.
template <bool kSkip>
__device__ __forceinline__ bool skipped(const DecodeParams& p, int s) {
    return kSkip && p.skip_seq[s] != 0;
}

// Item k of this CTA (k = 0, 1, ...).
template <bool kPersist, bool kSkip>
__device__ __forceinline__ Item get_item(const DecodeParams& p,
                                         const int* prefix, int k) {
    Item it;
    it.s = -1;
    int s, part;
    if (kPersist) {
        const int j = blockIdx.y + k * gridDim.y;
        if (j >= prefix[p.num_seqs]) return it;
        int lo = 0, hi = p.num_seqs - 1;  // largest s with prefix[s] <= j
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (prefix[mid] <= j) lo = mid; else hi = mid - 1;
        }
        s = lo;
        part = j - prefix[s];
    } else {
        if (k > 0) return it;
        s = blockIdx.z;
        part = blockIdx.y;
    }
    if (skipped<kSkip>(p, s)) return it;
    const int L = clamped_len(p, s);
    const int np = parts_of(L, p.partition_size);
    if (part >= np) return it;
    it.s = s;
    it.part = part;
    it.L = L;
    it.nparts = np;
    it.tok0 = part * p.partition_size;
    it.tok1 = min(L, it.tok0 + p.partition_size);
    return it;
}

// Chunks of `it` that warp w owns.
__device__ __forceinline__ int warp_chunks(const Item& it, int warp) {
    if (it.s < 0) return 0;
    const int n = (it.tok1 - it.tok0 + kChunk - 1) / kChunk;
    return n > warp ? (n - warp + kWarps - 1) / kWarps : 0;
}

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

template <int D, int BS, bool kPersist, bool kSkip>
__global__ void __launch_bounds__(kThreads, kTargetCtasPerSM)
paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const DecodeParams p) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char* ring = smem;
    float* red_o = reinterpret_cast<float*>(smem + C::kRedOff);
    float* red_m = red_o + (kWarps - 1) * kMaxGroup * C::kRedStride;
    float* red_l = red_m + kWarps * kMaxGroup;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    int* prefix = reinterpret_cast<int*>(smem + C::kPrefixOff);

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

    if (kPersist) {
        // prefix[s] = partitions of sequences 0..s-1 (block-wide scan).  The
        // merge area is free until the first item ends; it holds the warp sums.
        int* warp_tot = reinterpret_cast<int*>(red_l);
        int running = 0;
        if (threadIdx.x == 0) prefix[0] = 0;
        for (int base = 0; base < p.num_seqs; base += kThreads) {
            const int s = base + threadIdx.x;
            int v = 0;
            if (s < p.num_seqs && !skipped<kSkip>(p, s))
                v = parts_of(clamped_len(p, s), p.partition_size);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += t;
            }
            if (lane == 31) warp_tot[warp] = v;
            __syncthreads();
            int before = running;
            for (int w = 0; w < warp; ++w) before += warp_tot[w];
            if (s < p.num_seqs) prefix[s + 1] = before + v;
            for (int w = 0; w < kWarps; ++w) running += warp_tot[w];
            __syncthreads();
        }
    }

    uint64_t* my_bars = bars + warp * C::kStages;
    unsigned char* my_ring = ring + warp * C::kStages * C::kStageBytes;
    if (lane == 0) {
        for (int i = 0; i < C::kStages; ++i) mbar_init(&my_bars[i], 1);
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
    int prod_k = 0;        // item of the next chunk to look up
    int prod_i = 0;        // warp-chunk index within that item
    int prod_count = 0;    // chunks issued so far
    int ids_base = 0;      // prod_count at the last refill
    int ids = -1;          // lane l: slot coordinate of chunk ids_base + l
    bool prod_done = false;

    // Lane l finds the (ids_base + l)-th chunk of the stream and its slot.
    auto refill = [&]() {
        int k = prod_k, i = prod_i, n = lane;
        Item it = get_item<kPersist, kSkip>(p, prefix, k);
        for (;;) {
            if (it.s < 0) break;
            const int rem = warp_chunks(it, warp) - i;
            if (rem > n) break;
            n -= rem > 0 ? rem : 0;
            ++k;
            i = 0;
            it = get_item<kPersist, kSkip>(p, prefix, k);
        }
        int slot = -1;
        if (it.s >= 0) {
            i += n;
            const int ctok = it.tok0 + (warp + kWarps * i) * kChunk;
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
        prod_k = __shfl_sync(0xffffffffu, k, 31);
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
    int k = 0;
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
    Item next_it = get_item<kPersist, kSkip>(p, prefix, 0);
    uint32_t qnext[D / 16][2];
    load_q(next_it, qnext);
    for (;; ++k) {
        const Item it = next_it;
        if (it.s < 0) break;
        const int my_n = warp_chunks(it, warp);
        uint32_t qa[D / 16][2];
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = qnext[ks][0];
            qa[ks][1] = qnext[ks][1];
        }
        next_it = get_item<kPersist, kSkip>(p, prefix, k + 1);
        load_q(next_it, qnext);

        float o[D / 8][4];
#pragma unroll
        for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        float m_run = -INFINITY;
        float l_run = 0.f;

        for (int i = 0; i < my_n; ++i) {
            const int stage = cons_count % C::kStages;
            if (!aborted) {
                const bool ok = mbar_wait_bounded(&my_bars[stage],
                                                  (cons_count / C::kStages) & 1);
                if (!__all_sync(0xffffffffu, ok)) {
                    aborted = true;
                    drain_from = cons_count;
                    if (lane == 0) report(p.error_flags, PA_DEVERR_TIMEOUT);
                }
            }
            ++cons_count;
            if (aborted) continue;

            const int ctok = it.tok0 + (warp + kWarps * i) * kChunk;
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

        // ---------------- item end: merge the four warps ----------------
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
        if (warp != 0) {
            if (k > 0) named_bar_sync(2);  // warp 0 has read the previous item
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
                const bool direct = it.nparts == 1;
                const int64_t row = (int64_t)it.s * Hq + h;
                const int64_t idx = row * p.max_partitions + it.part;
                float* dst = direct ? p.out + row * D : p.tmp_o + idx * D;
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
                if (!direct && (lane & 3) == 0) {
                    p.tmp_m[idx] = M;
                    p.tmp_l[idx] = den;
                }
            }
            named_bar_arrive(2);
        }
    }
    // Consume warp 0's last "merged" arrival so no barrier is left pending.
    if (warp != 0 && k > 0) named_bar_sync(2);

    if (aborted) {
        // Drain copies still in flight on this warp's ring (bounded) before
        // the CTA exits.
        for (int c = drain_from; c < prod_count; ++c)
            (void)mbar_wait_bounded(&my_bars[c % C::kStages], (c / C::kStages) & 1);
    }
}

// Merge of the per-partition results: out = sum_p w_p o_p / sum_p w_p with
// w_p = l_p * 2^(m_p - max_p m_p).  One CTA of 8 warps per (query head,
// sequence); warp w takes partitions w, w+8, ... with 8 partitions' rows in
// flight per round, each lane holding D/32 consecutive columns.
constexpr int kReduceWarps = 8;
constexpr int kReduceUnroll = 8;

template <int D>
__global__ void __launch_bounds__(kReduceWarps * 32)
paged_decode_reduce_kernel(const DecodeParams p) {
    constexpr int V = D / 32;  // columns per lane
    const int h = blockIdx.x;
    const int s = blockIdx.y;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    pdl_wait();  // the partials come from the grid launched just before
    int L = p.context_lens[s];
    L = L < 0 ? 0 : (L > p.max_context_len ? p.max_context_len : L);
    if (p.skip_seq != nullptr && p.skip_seq[s] != 0) return;  // answered elsewhere
    const int np = (L + p.partition_size - 1) / p.partition_size;
    if (np <= 1) return;  // written directly by the partition kernel
    const int64_t base = ((int64_t)s * p.num_heads + h) * p.max_partitions;

    __shared__ float warp_max[kReduceWarps];
    __shared__ float part_acc[kReduceWarps][D];
    __shared__ float part_den[kReduceWarps];

    float M = -INFINITY;
    for (int i = threadIdx.x; i < np; i += kReduceWarps * 32)
        M = fmaxf(M, p.tmp_m[base + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) warp_max[warp] = M;
    __syncthreads();
    M = warp_max[0];
#pragma unroll
    for (int w = 1; w < kReduceWarps; ++w) M = fmaxf(M, warp_max[w]);

    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;
    float den = 0.f;
    for (int i0 = warp; i0 < np; i0 += kReduceWarps * kReduceUnroll) {
        float wts[kReduceUnroll];
        float vals[kReduceUnroll][V];
        float lv[kReduceUnroll], mv[kReduceUnroll];
#pragma unroll
        for (int u = 0; u < kReduceUnroll; ++u) {
            // Rows past np re-read the last row with weight 0, so every load
            // of the round is unconditional and in flight together.
            const int i = min(i0 + u * kReduceWarps, np - 1);
            lv[u] = p.tmp_l[base + i];
            mv[u] = p.tmp_m[base + i];
            const float* row = p.tmp_o + (base + i) * D + lane * V;
            if (V == 4) {
                const float4 t = *reinterpret_cast<const float4*>(row);
                vals[u][0] = t.x; vals[u][V > 1 ? 1 : 0] = t.y;
                vals[u][V > 2 ? 2 : 0] = t.z; vals[u][V > 3 ? 3 : 0] = t.w;
            } else {
                const float2 t = *reinterpret_cast<const float2*>(row);
                vals[u][0] = t.x; vals[u][V > 1 ? 1 : 0] = t.y;
            }
        }
#pragma unroll
        for (int u = 0; u < kReduceUnroll; ++u)
            wts[u] = i0 + u * kReduceWarps < np ? lv[u] * exp2f(mv[u] - M) : 0.f;
#pragma unroll
        for (int u = 0; u < kReduceUnroll; ++u) {
            den += wts[u];
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] += wts[u] * vals[u][v];
        }
    }
#pragma unroll
    for (int v = 0; v < V; ++v) part_acc[warp][lane * V + v] = acc[v];
    if (lane == 0) part_den[warp] = den;
    __syncthreads();
    for (int d = threadIdx.x; d < D; d += kReduceWarps * 32) {
        float a = 0.f, dn = 0.f;
#pragma unroll
        for (int w = 0; w < kReduceWarps; ++w) {
            a += part_acc[w][d];
            dn += part_den[w];
        }
        p.out[((int64_t)s * p.num_heads + h) * D + d] = a / dn;
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

template <int D, int BS, bool kSkip>
cudaError_t launch_partition_kernel(const DecodeParams& p, const CUtensorMap& tmk,
                                    const CUtensorMap& tmv, cudaStream_t stream) {
    using C = Cfg<D>;
    static int grid_ready[64] = {0};
    static int persist_ready[64] = {0};
    // Persistent CTAs when sequences are split, and when some sequences are
    // skipped (the compact item list then spends no CTA on them).
    const bool persist = (p.max_partitions > 1 || kSkip) && p.num_seqs <= kMaxPersistSeqs;
    cudaError_t e;
    if (persist) {
        e = set_smem(paged_decode_kernel<D, BS, true, kSkip>, C::kSmemPersist, persist_ready);
        if (e != cudaSuccess) return e;
        long long per_head = (kTargetCtasPerSM * kNumSMs + p.num_kv_heads - 1) / p.num_kv_heads;
        const long long items = (long long)p.num_seqs * p.max_partitions;
        if (per_head > items) per_head = items;
        if (per_head < 1) per_head = 1;
        dim3 grid((unsigned)p.num_kv_heads, (unsigned)per_head, 1);
        e = launch_pdl(paged_decode_kernel<D, BS, true, kSkip>, grid, dim3(kThreads),
                       C::kSmemPersist, stream, tmk, tmv, p);
    } else {
        e = set_smem(paged_decode_kernel<D, BS, false, kSkip>, C::kSmemGrid, grid_ready);
        if (e != cudaSuccess) return e;
        dim3 grid((unsigned)p.num_kv_heads, (unsigned)p.max_partitions,
                  (unsigned)p.num_seqs);
        e = launch_pdl(paged_decode_kernel<D, BS, false, kSkip>, grid, dim3(kThreads),
                       C::kSmemGrid, stream, tmk, tmv, p);
    }
    count_launch();
    return e;
}

template <int D, int BS>
cudaError_t launch_typed(const DecodeParams& p, cudaStream_t stream) {
    CUtensorMap tmk, tmv;
    if (!encode_pool_map(&tmk, p.k_cache, p.num_blocks, BS, p.num_kv_heads, D) ||
        !encode_pool_map(&tmv, p.v_cache, p.num_blocks, BS, p.num_kv_heads, D))
        return cudaErrorInvalidValue;
    cudaError_t e = p.skip_seq != nullptr
                        ? launch_partition_kernel<D, BS, true>(p, tmk, tmv, stream)
                        : launch_partition_kernel<D, BS, false>(p, tmk, tmv, stream);
    if (e != cudaSuccess) return e;
    if (p.max_partitions > 1) {
        dim3 rgrid((unsigned)p.num_heads, (unsigned)p.num_seqs);
        e = launch_pdl(paged_decode_reduce_kernel<D>, rgrid,
                       dim3(kReduceWarps * 32), 0, stream, p);
        count_launch();
    }
    return e;
}

}  // namespace

float log2e_scale(float scale) { return scale * kLog2e; }

cudaError_t launch_paged_decode(const DecodeParams& p, int head_size,
                                int block_size, cudaStream_t stream) {
    if (head_size == 128 && block_size == 16) return launch_typed<128, 16>(p, stream);
    if (head_size == 128 && block_size == 32) return launch_typed<128, 32>(p, stream);
    if (head_size == 64 && block_size == 16) return launch_typed<64, 16>(p, stream);
    if (head_size == 64 && block_size == 32) return launch_typed<64, 32>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
