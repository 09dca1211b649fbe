// Multi-query paged attention on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory) for tiles of 128 (query token, query head)
// rows: the chunked-prefill regime, where the work per KV byte is high enough
// for the contraction to be dense ("vLLM: Anatomy and Mechanisms of
// High-Throughput LLM Inference", "Chunked Prefill"; causal semantics as in
// pa_multi_query.cu).
//
// CTA = (kv head, 128-row tile, sequence), one per SM, 12 warps:
//   warps 0-7  softmax and epilogue in two warpgroups: warp w owns tile rows
//              32(w%4).. (its TMEM lane quarter); warpgroup 0 takes tokens
//              0-63 of each 128-token chunk and d 0-63 of the output,
//              warpgroup 1 tokens 64-127 and d 64-127.  Warps w and w+4 share
//              rows and agree per chunk through one named barrier (bar.red);
//   warps 8,10 producers of the K and the V stream: the tile's causal range
//              in 128-token chunks of 16-row TMA tensor tiles (128-byte
//              swizzle), one issuing thread per stream, 3- and 4-stage rings;
//   warp 9     allocates all 512 TMEM columns and issues the S MMAs,
//   warp 11    issues the PV MMAs (one thread each, descriptors built once).
//              The tensor pipe queues few MMAs, so a single issuing thread
//              left it idle during its waits between batches; with two, one
//              issues while the other waits.
// The 32 row tiles of a (sequence, kv head) read the same K and V, so the
// copies keep the default L2 priority (the decode stream's evict-first
// hint would send every tile back to DRAM).
//
// TMEM: S0 | S1 | O | Q (128, 128, 128, 64 columns).  Per chunk c:
// S(c) = Q K(c)^T (M=128, N=128, K=128: 8 tcgen05.mma, Q read from TMEM so
// that only K crosses shared memory) lands in buffer c%2; each warpgroup
// reads its 64 columns and writes P = bf16(p) and its bf16 residual back
// into them, and O += P V(c) runs as 2 x 8 tcgen05.mma with A read from
// TMEM (M=128, N=128, K=16 each).  S(c+1) is issued before PV(c), so the
// tensor core computes the next logits while the softmax warps work; S(c+2)
// waits until PV(c) has read the P it overwrites.
//
// Softmax reference.  The row max is taken exactly on the first chunk only;
// later chunks exponentiate against that reference and check the chunk's
// sum instead of taking a max: a sum above 2^16 (or not finite) means the
// row's max has grown, and only then are the logits (still in TMEM) read
// again, the exact max taken, O and the running sum rescaled and the chunk
// exponentiated afresh.  The sum and O share the reference, so the final
// O / l is exact; p <= 2^16 keeps the fp32 accumulator far from overflow.
// All waits are bounded, and the two warps of a row pair take every
// abort decision together; TMEM is released on every exit path.
#include <cuda.h>

#include <cstdint>
#include <mutex>

#include "pa_common.cuh"
#include "pa_multi_query.cuh"
#include "pa_split.cuh"

namespace pa {
namespace {

constexpr int kRows = 128;        // M: tile rows
constexpr int kTok = 128;         // tokens per chunk (N of S, K of PV)
constexpr int kD = 128;           // head size handled by this kernel
constexpr int kKStages = 3;
constexpr int kVStages = 4;
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = (kSoftmaxWarps + 4) * 32;  // + K, S, V, PV warps
constexpr int kWarpK = kSoftmaxWarps;
constexpr int kWarpMma = kSoftmaxWarps + 1;         // TMEM owner, S MMAs
constexpr int kWarpV = kSoftmaxWarps + 2;
constexpr int kWarpPv = kSoftmaxWarps + 3;
constexpr int kPiecesPerChunk = kTok / 16;          // 16-token TMA tiles
constexpr int kKVHalf = kTok * 128;                 // 16 KB: 128 tokens x 64 d
constexpr int kStageBytes = 2 * kKVHalf;            // one chunk of K or of V
constexpr int kKOff = 0;
constexpr int kVOff = kKOff + kKStages * kStageBytes;
constexpr int kXOff = kVOff + kVStages * kStageBytes;  // float [2][2][128]
constexpr int kBarOff = kXOff + 2 * 2 * kRows * 4;
// barriers: k_full[3], k_empty[3], v_full[4], v_empty[4], s_full[2],
//           p_full[2], pv_done[2] (per S buffer), o_final, q_ready, s_drain,
//           then the TMEM base address and the abort flag.  K and V travel
//           in separate rings: K(c) is free as soon as S(c) is done, long
//           before PV(c).
constexpr int kNumBars = 2 * kKStages + 2 * kVStages + 9;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
// Descriptor start addresses are 14-bit fields of (address >> 4).
static_assert(kSmemBytes + 1024 <= (1 << 18), "descriptor address range");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 2 * kTok;
constexpr uint32_t kTmemQ = kTmemO + kD;
constexpr float kSumLimit = 65536.f;                // 2^16: see the header

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

// 2^x by the PTX ex2.approx.ftz.f32 instruction (one MUFU operation):
// relative error about 2^-22, 2^-inf = 0, results below 2^-126 flush to 0
// (a term that small against the row's reference is invisible in fp32).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Pairs of fp32 values in one 64-bit register pair, for the sm_100 packed
// fp32 arithmetic (same rounding as the scalar instructions).
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// L2 policy with the default (normal) eviction priority.
__device__ __forceinline__ uint64_t l2_policy_normal() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
    return pol;
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

// Named barrier over the two warps (w, w + 4) that share tile rows, with an
// OR of their predicates.
__device__ __forceinline__ bool pair_any(int id, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, %2, 64, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void pair_sync(int id) {
    asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}

template <int BS>
__global__ void __launch_bounds__(kThreads, 1)
paged_multi_query_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v,
                            const MultiQueryParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* k_full = bars;
    uint64_t* k_empty = k_full + kKStages;
    uint64_t* v_full = k_empty + kKStages;
    uint64_t* v_empty = v_full + kVStages;
    uint64_t* s_full = v_empty + kVStages;
    uint64_t* p_full = s_full + 2;
    uint64_t* pv_done = p_full + 2;
    uint64_t* o_final = pv_done + 2;
    uint64_t* q_ready = o_final + 1;
    uint64_t* s_drain = q_ready + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
    int* abort_flag = reinterpret_cast<int*>(smem + kBarOff + kNumBars * 8 + 4);
    // Per-row exchange between the two warpgroups: [0] maxima, [1] sums.
    float (*xchg)[2][kRows] = reinterpret_cast<float (*)[2][kRows]>(smem + kXOff);

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
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < kVStages; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], kSoftmaxWarps * 32);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(o_final, 1);
        mbar_init(q_ready, kSoftmaxWarps * 32);
        mbar_init(s_drain, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == kWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + kTmemO;
    const uint32_t tmem_q = tmem + kTmemQ;

    if (warp == kWarpK || warp == kWarpV) {
        // --------------------------------------------------------- producers
        const int which = warp == kWarpV;               // 0: K, 1: V
        const int S = which ? kVStages : kKStages;
        uint64_t* fulls = which ? v_full : k_full;
        uint64_t* empties = which ? v_empty : k_empty;
        const int ring_off = which ? kVOff : kKOff;
        const uint64_t pol = l2_policy_normal();
        const int32_t* bt = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
        // Lane l holds the slot of 16-token piece l of chunks base..base+3.
        constexpr int kWindow = 32 / kPiecesPerChunk;   // chunks per window
        int piece_slot = -1;
        int slot_base = -kWindow;
        int issued = 0;
        for (int c = 0; c < nch; ++c, ++issued) {
            const int st = c % S;
            if (c >= S) {
                bool ok = true;
                if (lane == 0) ok = wait_bar(&empties[st], (c / S - 1) & 1);
                if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) {
                    if (lane == 0) set_abort(abort_flag, p.error_flags);
                    break;
                }
            }
            if (aborted(abort_flag)) break;
            if (c >= slot_base + kWindow) {
                slot_base = c - c % kWindow;
                const int t0 = slot_base * kTok + lane * 16;
                int v = -1;
                if (t0 < range_end) {
                    int id = bt[t0 / BS];
                    if (id < 0 || id >= p.num_blocks) {
                        report(p.error_flags, PA_DEVERR_BLOCK_ID);
                        id = 0;
                    }
                    v = id * BS + t0 % BS;
                }
                piece_slot = v;
            }
            int sl[kPiecesPerChunk];
#pragma unroll
            for (int i = 0; i < kPiecesPerChunk; ++i)
                sl[i] = __shfl_sync(0xffffffffu, piece_slot,
                                    (c - slot_base) * kPiecesPerChunk + i);
            if (lane == 0) {
                int pieces = 0;
#pragma unroll
                for (int i = 0; i < kPiecesPerChunk; ++i) pieces += sl[i] >= 0;
                const uint32_t base = smem_u32(smem + ring_off + st * kStageBytes);
                mbar_arrive_expect_tx(&fulls[st], pieces * 2 * 2048);
#pragma unroll
                for (int i = 0; i < kPiecesPerChunk; ++i) {
                    if (sl[i] < 0) continue;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tma_load(base + h * kKVHalf + i * 2048, which ? &tm_v : &tm_k,
                                 g * 2 + h, sl[i], &fulls[st], pol);
                }
            }
            __syncwarp();
        }
        // Wait for the copies still in flight before the CTA may exit.
        if (lane == 0)
            for (int c = (issued > S ? issued - S : 0); c < issued; ++c)
                (void)wait_bar(&fulls[c % S], (c / S) & 1);
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------ S MMA issuer
        constexpr uint32_t idesc_s = instr_desc(kRows, kTok, false);
        // K: K-major, its two 64-wide swizzle columns kKVHalf apart, 8-token
        // groups 1 KB apart; a 16-wide d slice starts 32 B into the 128-byte
        // row.  Each MMA adds a compile-time offset (16-byte units) to the
        // start-address field.
        const uint64_t k_desc0 = smem_desc(smem_u32(smem + kKOff), 16, 1024);
        bool ok = true;
        if (lane == 0) ok = wait_bar(q_ready, 0);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok && lane == 0) set_abort(abort_flag, p.error_flags);
        for (int c = 0; c < nch && ok; ++c) {
            const int ks_stage = c % kKStages;
            const int st = c & 1;
            bool good = true;
            if (lane == 0) {
                good = wait_bar(&k_full[ks_stage], (c / kKStages) & 1);
                // Buffer st holds P(c-2) until PV(c-2) has read it.
                if (good && c >= 2) good = wait_bar(&pv_done[st], ((c - 2) >> 1) & 1);
            }
            good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
            if (!good || aborted(abort_flag)) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint64_t kd = k_desc0 + (uint64_t)((ks_stage * kStageBytes) >> 4);
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t k_off = ((ks >> 2) * kKVHalf + (ks & 3) * 32) >> 4;
                    mma_ts(tmem + st * kTok, tmem_q + ks * 8, kd + k_off, idesc_s,
                           ks > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[st]);
                mma_commit(&k_empty[ks_stage]);
            }
            __syncwarp();
        }
        if (lane == 0) {
            mma_commit(s_drain);                 // this thread's MMAs retired
            (void)wait_bar(s_drain, 0);          // before TMEM goes away
        }
        __syncwarp();
    } else if (warp == kWarpPv) {
        // ----------------------------------------------------- PV MMA issuer
        constexpr uint32_t idesc_pv = instr_desc(kRows, kD, true);
        // V: MN-major, its two 64-wide d columns kKVHalf apart (LBO), 8-token
        // groups 1 KB apart (SBO).
        const uint64_t v_desc0 = smem_desc(smem_u32(smem + kVOff), kKVHalf, 1024);
        for (int c = 0; c < nch; ++c) {
            const int vs = c % kVStages;
            const int st = c & 1;
            // Every lane observes V(c) landing (the tail chunk's lanes write
            // into this stage below).
            bool good = __all_sync(0xffffffffu, wait_bar(&v_full[vs], (c / kVStages) & 1));
            if (good && lane == 0) good = wait_bar(&p_full[st], (c >> 1) & 1);
            good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
            if (!good || aborted(abort_flag)) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                break;
            }
            const int valid = min(kTok, range_end - c * kTok);
            if (valid < kTok) {
                // Rows past the range hold stale or unwritten data: zero the
                // V rows (P is 0 there, but 0 x NaN is NaN).
                unsigned char* vrow = smem + kVOff + vs * kStageBytes;
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
                const uint64_t vd = v_desc0 + (uint64_t)((vs * kStageBytes) >> 4);
                // P of tokens 16kt..16kt+15: warpgroup kt/4's 64 columns,
                // bf16 pairs at 8(kt%4), residuals 32 columns further.
                const uint32_t pb = tmem + st * kTok;
#pragma unroll
                for (int kt = 0; kt < kTok / 16; ++kt)
                    mma_ts(tmem_o, pb + 64 * (kt >> 2) + 8 * (kt & 3),
                           vd + (uint64_t)((kt * 2048) >> 4), idesc_pv,
                           (c > 0 || kt > 0) ? 1u : 0u);
#pragma unroll
                for (int kt = 0; kt < kTok / 16; ++kt)
                    mma_ts(tmem_o, pb + 64 * (kt >> 2) + 32 + 8 * (kt & 3),
                           vd + (uint64_t)((kt * 2048) >> 4), idesc_pv, 1u);
                mma_commit(&v_empty[vs]);
                mma_commit(&pv_done[st]);
            }
            __syncwarp();
        }
        if (lane == 0) {
            mma_commit(o_final);                 // every PV issued so far
            (void)wait_bar(o_final, 0);          // drained before TMEM goes away
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax, epilogue
        const int wg = warp >> 2;                // token half and d half
        const int qw = warp & 3;                 // TMEM lane quarter
        const int pair = 1 + qw;                 // named barrier of (w, w+4)
        const int r = qw * 32 + lane;            // tile row == TMEM lane
        const int R = row0 + r;
        const bool live = R < rows_total;
        const int j = live ? R / G : 0;
        const int gi = live ? R % G : 0;
        const int lim = live ? L - k + j : range_end - 1;
        const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
        const int col0 = 64 * wg;

        // This row's half of Q -> TMEM (the S MMA's A operand): column c
        // holds the bf16 pair (2c, 2c+1), the order of the words in memory.
        {
            const uint4* src = reinterpret_cast<const uint4*>(
                p.q + ((int64_t)(q0 + j) * Hq + g * G + gi) * kD + col0);
            uint32_t w[32];
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) {
                const uint4 v = live ? src[c16] : make_uint4(0, 0, 0, 0);
                w[4 * c16] = v.x;
                w[4 * c16 + 1] = v.y;
                w[4 * c16 + 2] = v.z;
                w[4 * c16 + 3] = v.w;
            }
            tmem_st32(tmem_q + lane_off + 32 * wg, w);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive_plain(q_ready);
        }

        const float sl2 = p.scale_log2;
        float m_ref = 0.f;
        float l_part = 0.f;
        bool ok = true;
        // Raw logits of this warpgroup's 64 tokens of chunk c from TMEM,
        // tokens past the row's causal limit set to -inf.  The scale (log2
        // domain) folds into one FFMA per exponent; maxima are taken on raw
        // values and scaled (scale > 0 preserves order).
        auto load_logits = [&](uint32_t sbase, int ctok, float (&sv)[64]) {
            uint32_t r0[32], r1[32];
            tmem_ld32(sbase, r0);
            tmem_ld32(sbase + 32, r1);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                sv[i] = __uint_as_float(r0[i]);
                sv[32 + i] = __uint_as_float(r1[i]);
            }
            if (ctok + 63 > min_lim) {
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (ctok + i > lim) sv[i] = -INFINITY;
            }
        };
        auto half_max = [&](const float (&sv)[64]) -> float {
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = sv[i];
#pragma unroll
            for (int i = 8; i < 64; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], sv[i]);
            return sl2 * fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        };
        // In place: sv <- 2^(scale*s - m_ref) (masked logits give 0); the sum.
        // The exponent arguments and the partial sums run on pairs
        // (fma.rn.f32x2 / add.rn.f32x2: the scalar roundings, half the
        // instructions).
        auto exponentiate = [&](float (&sv)[64]) -> float {
            const uint64_t s2 = pack_f32x2(sl2, sl2);
            const uint64_t nm2 = pack_f32x2(-m_ref, -m_ref);
            uint64_t acc[4] = {0, 0, 0, 0};      // four packed pairs of partial sums
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float a, b;
                unpack_f32x2(fma_f32x2(pack_f32x2(sv[2 * i], sv[2 * i + 1]), s2, nm2), a, b);
                sv[2 * i] = ex2_approx(a);
                sv[2 * i + 1] = ex2_approx(b);
                acc[i & 3] = add_f32x2(acc[i & 3], pack_f32x2(sv[2 * i], sv[2 * i + 1]));
            }
            float ps8[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) unpack_f32x2(acc[j], ps8[2 * j], ps8[2 * j + 1]);
            return ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) +
                   ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
        };
        for (int c = 0; c < nch; ++c) {
            const int st = c & 1;
            const bool got = wait_bar(&s_full[st], (c >> 1) & 1);
            if (pair_any(pair, !got || aborted(abort_flag))) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sbase = tmem + lane_off + st * kTok + col0;
            const int ctok = c * kTok + col0;
            float sv[64];
            load_logits(sbase, ctok, sv);
            if (c == 0) {                        // token 0 is visible to every row
                xchg[0][wg][r] = half_max(sv);
                pair_sync(pair);
                m_ref = fmaxf(xchg[0][0][r], xchg[0][1][r]);
            }
            float psum = exponentiate(sv);
            if (pair_any(pair, !(psum <= kSumLimit))) {
                // A row's max grew: exact max from the logits still in TMEM,
                // O and the sums rescaled once the previous PV is done.
                load_logits(sbase, ctok, sv);
                xchg[0][wg][r] = half_max(sv);
                pair_sync(pair);
                const float m_new = fmaxf(m_ref, fmaxf(xchg[0][0][r], xchg[0][1][r]));
                if (c > 0) {
                    const bool okw = wait_bar(&pv_done[(c - 1) & 1], ((c - 1) >> 1) & 1);
                    if (pair_any(pair, !okw)) {
                        if (lane == 0) set_abort(abort_flag, p.error_flags);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float alpha = exp2f(m_ref - m_new);
                    l_part *= alpha;
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        uint32_t o[32];
                        tmem_ld32(tmem_o + lane_off + col0 + part * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(tmem_o + lane_off + col0 + part * 32, o);
                    }
                    tmem_wait_st();
                }
                m_ref = m_new;
                psum = exponentiate(sv);
            }
            l_part += psum;
            // p as bf16 plus its bf16 residual, both rounded to nearest (P
            // carries ~17 bits into PV).  Pairs of tokens in the
            // warpgroup's first 32 columns, the residuals in the next 32.
            uint32_t hi[32], lo[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) split_bf16x2(sv[2 * i], sv[2 * i + 1], hi[i], lo[i]);
            tmem_st32(sbase, hi);
            tmem_st32(sbase + 32, lo);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive_plain(&p_full[st]);
        }
        if (ok) {
            xchg[1][wg][r] = l_part;
            const bool okw = wait_bar(o_final, 0);
            // Also orders the partner's sum before the read below.
            if (!pair_any(pair, !okw)) {
                tc_fence_after();
                float* dst = p.out + ((int64_t)(q0 + j) * Hq + g * G + gi) * kD + col0;
                const float inv = 1.f / (xchg[1][0][r] + xchg[1][1][r]);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint32_t o[32];
                    tmem_ld32(tmem_o + lane_off + col0 + part * 32, o);
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
    if (warp == kWarpMma)
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
