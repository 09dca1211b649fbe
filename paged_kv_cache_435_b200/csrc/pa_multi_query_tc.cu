// Multi-query paged attention on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory) for tiles of 128 (query token, query head)
// rows: the chunked-prefill regime, where the work per KV byte is high enough
// for the contraction to be dense ("vLLM: Anatomy and Mechanisms of
// High-Throughput LLM Inference", "Chunked Prefill"; causal semantics as in
// pa_multi_query.cu).
//
// CTA = (kv head, 128-row tile, sequence), 6 warps:
//   warps 0-3  softmax and epilogue; thread i owns tile row i, which is TMEM
//              lane i, so row max / row sum need no shuffles;
//   warp 4     producer: 64-token K/V chunks of the tile's causal range, as
//              16-row TMA tensor tiles (128-byte swizzle), into a 2-stage ring;
//   warp 5     allocates 256 TMEM columns and issues the MMAs (one thread).
// Per chunk c: S(c) = Q K(c)^T (M=128, N=64, K=128: 8 tcgen05.mma, both
// operands in shared memory) lands in TMEM buffer c%2; the softmax warps read
// their rows, write P = bf16(p) and its bf16 residual back into the same
// buffer, and O += P V(c) runs as 2 x 4 tcgen05.mma with A read from TMEM
// (M=128, N=128, K=16 each).  S(c+1) is issued before PV(c), so the tensor
// core computes the next logits while the softmax warps work.  O stays in
// TMEM (128 columns); it is rescaled only when a row's running max grows by
// more than 2^8 (the sum and O share the stale reference, so the final O/l is
// exact).  All waits are bounded; TMEM is released on every exit path.
#include <cuda.h>

#include <cstdint>
#include <mutex>

#include "pa_common.cuh"
#include "pa_multi_query.cuh"

namespace pa {
namespace {

constexpr int kRows = 128;        // M: tile rows
constexpr int kTok = 64;          // tokens per chunk (N of S, K of PV)
constexpr int kD = 128;           // head size handled by this kernel
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr int kQHalf = kRows * 128;                 // 16 KB: 128 rows x 64 d
constexpr int kKVHalf = kTok * 128;                 // 8 KB: 64 tokens x 64 d
constexpr int kStageBytes = 4 * kKVHalf;            // K lo/hi, V lo/hi
constexpr int kQOff = 0;
constexpr int kRingOff = 2 * kQHalf;                // 32 KB
constexpr int kBarOff = kRingOff + kStages * kStageBytes;
// barriers: k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2],
//           p_full[2], pv_done, o_final, q_ready, then the TMEM base address
//           and the abort flag.  K and V travel in separate rings: K(c) is
//           free as soon as S(c) is done, long before PV(c).
constexpr int kNumBars = 15;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16;
constexpr uint32_t kTmemCols = 256;                 // S0 | S1 | O
constexpr float kRescaleThreshold = 8.f;            // log2 units

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    return mbar_wait_bounded(bar, parity);
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo,
                                              uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // version
    d |= (uint64_t)2 << 61;   // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: fp32 D, bf16 A and B, A K-major.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc,
                                       uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate),
        "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem,
                                       uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate),
        "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
          "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
          "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]),
          "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]),
          "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]),
          "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
          "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),
          "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
          "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load(uint32_t dst, const CUtensorMap* map,
                                         int c1, int c2, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::"
        "complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(c1), "r"(c2),
        "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_plain(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void set_abort(int* flag, int* error_flags) {
    if (atomicExch(flag, 1) == 0) report(error_flags, PA_DEVERR_TIMEOUT);
}
__device__ __forceinline__ bool aborted(int* flag) {
    return *reinterpret_cast<volatile int*>(flag) != 0;
}

template <int BS>
__global__ void __launch_bounds__(kThreads, 2)
paged_multi_query_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v,
                            const MultiQueryParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* k_full = bars + 0;
    uint64_t* k_empty = bars + 2;
    uint64_t* v_full = bars + 4;
    uint64_t* v_empty = bars + 6;
    uint64_t* s_full = bars + 8;
    uint64_t* p_full = bars + 10;
    uint64_t* pv_done = bars + 12;
    uint64_t* o_final = bars + 13;
    uint64_t* q_ready = bars + 14;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
    int* abort_flag = reinterpret_cast<int*>(smem + kBarOff + kNumBars * 8 + 4);

    const int g = blockIdx.x;
    const int rt = blockIdx.y;
    const int s = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.group;
    const int Hq = p.num_heads;

    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) report(p.error_flags, PA_DEVERR_INTERNAL);
        return;
    }
    pdl_wait();
    pdl_launch_dependents();

    int L = p.context_lens[s];
    if (L < 0 || L > p.max_context_len) {
        if (threadIdx.x == 0 && g == 0 && rt == 0) report(p.error_flags, PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : p.max_context_len;
    }
    const int q0 = p.query_start_loc[s];
    int k = p.query_start_loc[s + 1] - q0;
    if (k < 0 || k > L || k > p.max_query_len) {
        if (threadIdx.x == 0 && g == 0 && rt == 0) report(p.error_flags, PA_DEVERR_QUERY_LEN);
        k = k < 0 ? 0 : min(k, min(L, p.max_query_len));
    }
    const int rows_total = k * G;
    const int row0 = rt * kRows;
    if (row0 >= rows_total) return;
    const int j_hi = min(k - 1, (row0 + kRows - 1) / G);
    const int min_lim = L - k + row0 / G;
    const int range_end = L - k + j_hi + 1;            // tokens [0, range_end)
    const int nch = (range_end + kTok - 1) / kTok;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
        }
        mbar_init(pv_done, 1);
        mbar_init(o_final, 1);
        mbar_init(q_ready, 128);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + 2 * kTok;          // columns [128, 256)

    const uint64_t pol = l2_policy_evict_first();

    if (warp == 4) {
        // ---------------------------------------------------------- producer
        // Order: K(0), K(1), V(0), K(2), V(1), ...: V runs one chunk behind
        // K, so a K stage is refilled as soon as S has read it.
        const int32_t* bt = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
        // Per stream (K, V): lane l holds the slot of 16-token piece l of
        // chunks base..base+7 (V runs one chunk behind K, so each stream
        // keeps its own window).
        int piece_slot[2] = {-1, -1};
        int slot_base[2] = {-8, -8};
        auto slots_of = [&](int c, int which, int (&sl)[4]) {
            if (c >= slot_base[which] + 8) {
                slot_base[which] = c & ~7;
                const int t0 = slot_base[which] * kTok + lane * 16;
                int v = -1;
                if (t0 < range_end) {
                    int id = bt[t0 / BS];
                    if (id < 0 || id >= p.num_blocks) {
                        report(p.error_flags, PA_DEVERR_BLOCK_ID);
                        id = 0;
                    }
                    v = id * BS + t0 % BS;
                }
                piece_slot[which] = v;
            }
            const int mine = piece_slot[which];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                sl[i] = __shfl_sync(0xffffffffu, mine, (c - slot_base[which]) * 4 + i);
        };
        // Issue K (which = 0) or V (which = 1) of chunk c; false on abort.
        auto load = [&](int c, int which) -> bool {
            const int st = c & 1;
            uint64_t* full = which ? &v_full[st] : &k_full[st];
            uint64_t* empty = which ? &v_empty[st] : &k_empty[st];
            if (c >= kStages) {
                bool ok = true;
                if (lane == 0) ok = wait_bar(empty, ((c >> 1) - 1) & 1);
                if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) {
                    if (lane == 0) set_abort(abort_flag, p.error_flags);
                    return false;
                }
            }
            if (aborted(abort_flag)) return false;
            int sl[4];
            slots_of(c, which, sl);
            if (lane == 0) {
                int pieces = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) pieces += sl[i] >= 0;
                const uint32_t base = smem_u32(smem + kRingOff + st * kStageBytes +
                                               which * 2 * kKVHalf);
                mbar_arrive_expect_tx(full, pieces * 2 * 2048);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (sl[i] < 0) continue;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tma_load(base + h * kKVHalf + i * 2048, which ? &tm_v : &tm_k,
                                 g * 2 + h, sl[i], full, pol);
                }
            }
            __syncwarp();
            return true;
        };
        int k_issued = 0, v_issued = 0;
        for (int c = 0; c <= nch; ++c) {
            if (c < nch) {
                if (!load(c, 0)) break;
                ++k_issued;
            }
            if (c >= 1) {
                if (!load(c - 1, 1)) break;
                ++v_issued;
            }
        }
        // Wait for the copies still in flight before the CTA may exit.
        if (lane == 0) {
            for (int c = (k_issued > kStages ? k_issued - kStages : 0); c < k_issued; ++c)
                (void)wait_bar(&k_full[c & 1], (c >> 1) & 1);
            for (int c = (v_issued > kStages ? v_issued - kStages : 0); c < v_issued; ++c)
                (void)wait_bar(&v_full[c & 1], (c >> 1) & 1);
        }
    } else if (warp == 5) {
        // --------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc_s = instr_desc(kRows, kTok, false);
        constexpr uint32_t idesc_pv = instr_desc(kRows, kD, true);
        const uint32_t q_base = smem_u32(smem + kQOff);
        bool ok = true;
        if (lane == 0) ok = wait_bar(q_ready, 0);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok && lane == 0) set_abort(abort_flag, p.error_flags);
        int issued_pv = 0;
        auto issue_pv = [&](int c) -> bool {
            const int st = c & 1;
            // Every lane observes V(c) landing (the tail chunk's lanes write
            // into this stage below).
            bool good = __all_sync(0xffffffffu, wait_bar(&v_full[st], (c >> 1) & 1));
            if (good && lane == 0) good = wait_bar(&p_full[st], (c >> 1) & 1);
            good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
            if (!good) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                return false;
            }
            const int valid = min(kTok, range_end - c * kTok);
            if (valid < kTok) {
                // Rows past the range hold stale or unwritten data: zero the
                // V rows (P is 0 there, but 0 x NaN is NaN).
                unsigned char* vrow = smem + kRingOff + st * kStageBytes + 2 * kKVHalf;
                const int rows = kTok - valid;
                for (int e = lane; e < rows * 2 * 8; e += 32) {
                    const int r = valid + e / 16;
                    const int h = (e / 8) & 1;
                    *reinterpret_cast<uint4*>(vrow + h * kKVHalf + r * 128 + (e & 7) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t v_base = smem_u32(smem + kRingOff + st * kStageBytes + 2 * kKVHalf);
                const uint32_t p_hi = tmem + st * kTok;
                const uint32_t p_lo = p_hi + kTok / 2;
#pragma unroll
                for (int kt = 0; kt < kTok / 16; ++kt) {
                    // V rows 16kt..16kt+15 (two 8-row groups), MN-major:
                    // LBO = the 8 KB between the two 64-column halves.
                    const uint64_t vd = smem_desc(v_base + kt * 2048, kKVHalf, 1024);
                    mma_ts(tmem_o, p_hi + kt * 8, vd, idesc_pv, (c > 0 || kt > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kt = 0; kt < kTok / 16; ++kt) {
                    const uint64_t vd = smem_desc(v_base + kt * 2048, kKVHalf, 1024);
                    mma_ts(tmem_o, p_lo + kt * 8, vd, idesc_pv, 1u);
                }
                mma_commit(&v_empty[st]);
                mma_commit(pv_done);
            }
            __syncwarp();
            ++issued_pv;
            return true;
        };
        for (int c = 0; c < nch && ok; ++c) {
            const int st = c & 1;
            bool good = true;
            if (lane == 0) good = wait_bar(&k_full[st], (c >> 1) & 1);
            good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
            if (!good || aborted(abort_flag)) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t k_base = smem_u32(smem + kRingOff + st * kStageBytes);
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks & 3) * 32;  // K=16 slice in the atom
                    const uint64_t qd = smem_desc(q_base + (ks >> 2) * kQHalf + off, 16, 1024);
                    const uint64_t kd = smem_desc(k_base + (ks >> 2) * kKVHalf + off, 16, 1024);
                    mma_ss(tmem + st * kTok, qd, kd, idesc_s, ks > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[st]);
                mma_commit(&k_empty[st]);
            }
            __syncwarp();
            if (c >= 1 && !issue_pv(c - 1)) break;
        }
        if (!aborted(abort_flag) && issued_pv == nch - 1 && nch >= 1) issue_pv(nch - 1);
        if (lane == 0) {
            mma_commit(o_final);                 // everything issued so far
            (void)wait_bar(o_final, 0);          // drained before TMEM goes away
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax, epilogue
        const int r = warp * 32 + lane;          // tile row == TMEM lane
        const int R = row0 + r;
        const bool live = R < rows_total;
        const int j = live ? R / G : 0;
        const int gi = live ? R % G : 0;
        const int lim = live ? L - k + j : range_end - 1;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

        // Q row -> shared memory in the K-major 128-byte-swizzled layout.
        {
            const uint4* src = reinterpret_cast<const uint4*>(
                p.q + ((int64_t)(q0 + j) * Hq + g * G + gi) * kD);
#pragma unroll
            for (int c16 = 0; c16 < 16; ++c16) {
                const uint4 v = live ? src[c16] : make_uint4(0, 0, 0, 0);
                const int h = c16 >> 3, cc = c16 & 7;
                *reinterpret_cast<uint4*>(smem + kQOff + h * kQHalf + r * 128 +
                                          ((cc ^ (r & 7)) << 4)) = v;
            }
            fence_proxy_async_smem();
            mbar_arrive_plain(q_ready);
        }

        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY;
        float l_sum = 0.f;
        bool ok = true;
        for (int c = 0; c < nch; ++c) {
            const int st = c & 1;
            ok = wait_bar(&s_full[st], (c >> 1) & 1);
            if (!__all_sync(0xffffffffu, ok) || aborted(abort_flag)) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sraw[2][32];
            tmem_ld32(tmem + lane_off + st * kTok, sraw[0]);
            tmem_ld32(tmem + lane_off + st * kTok + 32, sraw[1]);
            tmem_wait_ld();
            // Raw logits; the scale (log2 domain) folds into one FFMA per
            // exponent below, and the row max is taken on raw values
            // (scale > 0 preserves order).
            float sv[64];
            const int ctok = c * kTok;
#pragma unroll
            for (int i = 0; i < 64; ++i) sv[i] = __uint_as_float(sraw[i >> 5][i & 31]);
            if (ctok + kTok - 1 > min_lim) {
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (ctok + i > lim) sv[i] = -INFINITY;
            }
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = sv[i];
#pragma unroll
            for (int i = 8; i < 64; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], sv[i]);
            const float mx = sl2 * fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            if (c == 0) {
                m_ref = mx;
            } else if (__any_sync(0xffffffffu, mx > m_ref + kRescaleThreshold)) {
                // O must be stable: the previous chunk's PV has to be done.
                const bool okw = wait_bar(pv_done, (c - 1) & 1);
                if (!__all_sync(0xffffffffu, okw)) {
                    if (lane == 0) set_abort(abort_flag, p.error_flags);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float m_new = fmaxf(m_ref, mx);
                const float alpha = exp2f(m_ref - m_new);
                m_ref = m_new;
                l_sum *= alpha;
#pragma unroll
                for (int part = 0; part < kD / 32; ++part) {
                    uint32_t o[32];
                    tmem_ld32(tmem_o + lane_off + part * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tmem_o + lane_off + part * 32, o);
                }
                tmem_wait_st();
            }
            // p = 2^(scale*s - m) (masked logits give 2^-inf = 0) and its bf16
            // split by truncation: the high half keeps 8 significant bits, the
            // residual another 8, so P carries ~16 bits into PV.
            uint32_t hi[32], lo[32];
            float ps8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            const float neg_m = -m_ref;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float a = exp2f(fmaf(sv[2 * i], sl2, neg_m));
                const float b = exp2f(fmaf(sv[2 * i + 1], sl2, neg_m));
                ps8[i & 7] += a + b;
                const uint32_t ab = __float_as_uint(a), bb = __float_as_uint(b);
                const float al = a - __uint_as_float(ab & 0xFFFF0000u);
                const float bl = b - __uint_as_float(bb & 0xFFFF0000u);
                hi[i] = __byte_perm(ab, bb, 0x7632);
                lo[i] = __byte_perm(__float_as_uint(al), __float_as_uint(bl), 0x7632);
            }
            l_sum += ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) +
                     ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
            tmem_st32(tmem + lane_off + st * kTok, hi);
            tmem_st32(tmem + lane_off + st * kTok + 32, lo);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive_plain(&p_full[st]);
        }
        if (ok) {
            const bool okw = wait_bar(o_final, 0);
            if (__all_sync(0xffffffffu, okw)) {
                tc_fence_after();
                float* dst = p.out + ((int64_t)(q0 + j) * Hq + g * G + gi) * kD;
                const float inv = 1.f / l_sum;
#pragma unroll
                for (int part = 0; part < kD / 32; ++part) {
                    uint32_t o[32];
                    tmem_ld32(tmem_o + lane_off + part * 32, o);
                    tmem_wait_ld();
                    if (live) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4*>(dst + part * 32 + i) = make_float4(
                                __uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                                __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                    }
                }
            } else if (lane == 0) {
                set_abort(abort_flag, p.error_flags);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                   void*, const cuuint64_t*, const cuuint64_t*,
                                   const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tc_encode_fn() {
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

bool tc_encode_map(CUtensorMap* map, const void* pool, int num_blocks,
                   int block_size, int num_kv_heads) {
    EncodeTiledFn fn = tc_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)num_kv_heads * kD / 64,
                                (cuuint64_t)num_blocks * block_size};
    const cuuint64_t strides[2] = {128, (cuuint64_t)num_kv_heads * kD * 2};
    const cuuint32_t box[3] = {64, 1, 16};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BS>
cudaError_t tc_launch_typed(const MultiQueryParams& p, cudaStream_t stream) {
    static int ready[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE)) {
        e = cudaFuncSetAttribute(paged_multi_query_tc_kernel<BS>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
    }
    CUtensorMap tmk, tmv;
    if (!tc_encode_map(&tmk, p.k_cache, p.num_blocks, BS, p.num_kv_heads) ||
        !tc_encode_map(&tmv, p.v_cache, p.num_blocks, BS, p.num_kv_heads))
        return cudaErrorInvalidValue;
    const int tiles = (p.max_query_len * p.group + kRows - 1) / kRows;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_kv_heads, (unsigned)tiles, (unsigned)p.num_seqs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, paged_multi_query_tc_kernel<BS>, tmk, tmv, p);
    count_launch();
    return e;
}

}  // namespace

bool multi_query_tc_eligible(int head_size, int max_query_len, int group) {
    return head_size == kD && (long long)max_query_len * group >= kRows;
}

cudaError_t launch_paged_multi_query_tc(const MultiQueryParams& p,
                                        int block_size, cudaStream_t stream) {
    if (block_size == 16) return tc_launch_typed<16>(p, stream);
    if (block_size == 32) return tc_launch_typed<32>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
