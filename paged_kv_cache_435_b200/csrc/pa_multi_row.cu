// Paged attention for up to 32 query rows per kv head on the tcgen05 tensor
// cores, with the operands swapped so that the tokens fill the MMA's M.
//
// Two callers share it:
//  * speculative verification (pa_multi_query_attention): the k proposed
//    tokens of a sequence times the G query heads of a kv head are the rows,
//    causal within the chunk ("vLLM: Anatomy and Mechanisms of
//    High-Throughput LLM Inference", "Speculative Decoding");
//  * the group pass of pa_decode_attention_shared_prefix: the samples of one
//    prompt times the G heads are the rows ("Memory Sharing via Copy-on-Write
//    (CoW)").  An item streams the prompt blocks the samples share once for
//    all rows, then each sample's private tail for that sample's rows only,
//    along one virtual token axis: [0, shared end) shared, then the tails,
//    each padded to 16 tokens; a row sees the shared tokens of its context
//    and its own tail.
// With 32 rows over a stream of KV the work is 32 flop per KV byte, far below
// the tensor roofline: the goal is to read every block once at HBM speed with
// the math hidden behind it.  A 128-row M tile would waste 3/4 of the tensor
// core on such a stream, so the products are transposed:
//     S^T (128 tokens x 32 rows)  = K (128 x 128 d) . Q^T (128 d x 32 rows)
//     O^T (128 d x 64)           += V^T (128 d x 128 tokens) . [P_hi^T | P_lo^T]
// with M = 128 in both.  K comes from its TMA tile as a K-major A operand, V
// as an MN-major A operand (the same tile, read transposed by the
// descriptor).  Q^T is a K-major B operand; P's bf16 high part and its bf16
// residual sit side by side as one MN-major B operand of N = 64 (one
// 128-byte row per token, written by that token's thread), so V is read
// once per chunk and O_hi, O_lo accumulate in adjacent TMEM columns, summed
// at the end.  Accumulators live in tensor memory: S^T double-buffered (2 x 32
// columns), O^T double-buffered across items (2 x 64 columns).
//
// CTA: 8 warps, one CTA per SM, persistent over items (row tile, kv head):
//   warps 0-3  softmax: thread i owns token i of the chunk (TMEM lane i) and
//              all 32 rows; P = 2^(s - m) as bf16 high part + bf16 residual
//              (~16 bits into the PV product), one 128-byte row of P^T;
//   warp 4     K producer, warp 5 V producer: 16-token TMA tensor tiles
//              (128-byte swizzle) of each 128-token chunk into 2- and 3-stage
//              rings (V waits for the softmax, so it runs deeper);
//   warp 6     TMEM allocation and the MMA issue (one thread), S two chunks
//              ahead of PV: S(n) needs only that the softmax has loaded
//              S(n-2) out of its TMEM buffer, PV(n-2) that it wrote P(n-2);
//   warp 7     scheduler: deals the items to the CTAs by work and publishes
//              them.  A CTA serves one kv head; the CTAs of a head take the
//              units (sequences or groups) longest first in snake order when
//              every unit is one item (a bitonic sort across the warp), else
//              the items whose cumulative weight starts in their share; all
//              heads walk the batch in the same order, so the head slices of
//              a block are read together.  In the group pass, when one item
//              alone is longer than 1.5 CTA shares, the items are instead cut
//              into pieces at 128-token chunk boundaries so that every CTA of
//              the head gets an even share; a piece writes its rows' partial
//              (reference, sum, normalised O) and the last piece of an item to
//              finish merges them into the output.  For each item or piece
//              it works out the token range, block-table rows, each row's
//              visible tokens, output row and reference into a 4-slot
//              shared-memory ring and copies the Q rows (cp.async), so no
//              other warp waits on a global load at an item boundary.
// Online softmax with a lazy reference: each row starts from its logit at
// its first visible token of the item or piece (so its sum is at least 1),
// which the scheduler computes (q . k of that token's K row) when it
// publishes the item; the row's tokens before that one are masked.  Every chunk,
// one barrier-reduction over the 4 warps (bar.red.popc) asks whether any
// row's logit exceeds its reference by more than 2^24 (weights stay below
// 2^24, far from fp32 overflow, and the split of P keeps its relative
// precision at any scale, so the reference need not be tight); only then is
// the exact per-row chunk max formed (warp transpose-reduction + shared
// memory), O^T rescaled in TMEM and the reference moved.  Sums are kept per
// thread and reduced at item end.
// A token no row may see (padding, past the range) has its V row zeroed by
// its own thread once the chunk landed: P is 0 there, but 0 x NaN is NaN.
// The producers and the MMA warp run ahead across item boundaries; the
// epilogue of an item runs one chunk into the next item.  Every wait is
// bounded; the softmax warps decide aborts together at their per-chunk
// barrier, and TMEM is released on every exit path.
#include <cuda.h>

#include <cstdint>
#include <mutex>

#include "pa_cascade.cuh"
#include "pa_common.cuh"
#include "pa_split.cuh"
#include "pa_multi_row.cuh"

namespace pa {
namespace {

constexpr int kTok = 128;                 // tokens per chunk (M of both products)
constexpr int kN = kMultiRowTile;         // rows (N of both products)
constexpr int kD = 128;
constexpr int kKStages = 2;
constexpr int kVStages = 3;
constexpr int kThreads = 256;
constexpr int kSlots = 4;                 // items published ahead by the scheduler
constexpr int kHalf = kTok * 128;         // 16 KB: 128 tokens x 64 d (one swizzle column)
constexpr int kStageBytes = 2 * kHalf;    // 32 KB: one chunk of K or V
constexpr int kQHalf = kN * 128;          // 4 KB: 32 rows x 64 d
constexpr int kQBytes = 2 * kQHalf;
constexpr int kPBytes = kTok * 128;       // 16 KB: P^T of a chunk, 128 B per token
constexpr int kKOff = 0;
constexpr int kVOff = kKOff + kKStages * kStageBytes;
constexpr int kQOff = kVOff + kVStages * kStageBytes;  // 2 item buffers
constexpr int kPOff = kQOff + 2 * kQBytes;             // 2 chunk buffers x (hi | lo)
constexpr int kMiscOff = kPOff + 2 * kPBytes;
constexpr int kCmaxOff = kMiscOff;                     // float [32][4]
// Largest unit weight the scheduler's counting sort handles (its histogram
// and order live in the P buffers before the first item is published).
constexpr int kCountSortMaxWeight = 2048;

// One published item: what every role needs, and the per-row results the
// epilogue writes out.
struct ItemSlot {
    int table_seq, g, range_end, nch;   // nch: one past the last chunk of this
                                        // piece (< 0: no further items)
    int c0;                             // first chunk of this piece
    int piece;                          // -1: the whole item (writes the
                                        // output); else its partial's slot
    int unit, item_n;                   // split item: group, its chunks
    int item_a, axis_len;               // split item: first position, axis
                                        // length (see the split deal)
    int pad0_;
    uint32_t live_rows;                 // rows that exist (bit r: row r)
    float m_fin[32], l_fin[32];         // rows: reference and sum at the end
    float ref[32];                      // rows: logit at the first visible token
                                        // of the piece (0: none), the scheduler's
    int min_lim, nmem, shared_r16, P;   // smallest row limit; members (group
                                        // mode); end of the shared region
                                        // rounded to 16; prefix length
    int arrived, pad_[3];               // pieces counted before this one
    int lim[32];                        // rows: last visible shared token
    int mem_tend[32];                   // members: end of the unpadded tail
    uint32_t mem_rows[32];              // members: their rows (bit r: row r)
    int mem_seq[32];                    // members: sequence
    int mem_v[32], mem_vend[32];        // members: tail pieces [v, vend)
    long long row[32];                  // q / out row of each row (-1: none)
    float red_l[32][4];                 // per-warp partial row sums
    float inv_l[32];                    // 1 / row sum (0 for an empty row)
};
static_assert(sizeof(ItemSlot) == 2128 && sizeof(ItemSlot) % 16 == 0, "slot layout");

constexpr int kSlotOff = kCmaxOff + 512;
constexpr int kBarOff = kSlotOff + kSlots * (int)sizeof(ItemSlot);
// barriers: k_full[KS] k_empty[KS] v_full[VS] v_empty[VS] s_full[2] s_free[2]
//           p_full[2] pv_done[2] o_full[2] o_empty[2] q_empty[2] item_ready[4]
//           slot_free[4] drain item_meta[4] item_refs[4]
constexpr int kNumBars = 2 * kKStages + 2 * kVStages + 15 + 4 * kSlots;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16;
constexpr uint32_t kTmemCols = 256;       // S0 | S1 | O0 (hi, lo) | O1 (hi, lo)
constexpr uint32_t kTmemO = 64;           // first O column
constexpr float kRescaleThreshold = 24.f;  // log2 units

static_assert((kCountSortMaxWeight + 1 + 256) * 4 <= 2 * kPBytes,
              "the scheduler's counting sort fits in the P buffers");
static_assert(kStageBytes % 1024 == 0 && kQBytes % 1024 == 0 && kPBytes % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
static_assert(kSlotOff % 16 == 0 && kBarOff % 8 == 0, "alignment");
static_assert(kSmemBytes <= 232448, "shared memory");
// Descriptor start addresses are 14-bit fields of (address >> 4); offsets
// are added to a base descriptor without a carry out of that field.
static_assert(kSmemBytes + 1024 <= (1 << 18), "descriptor address range");

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
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::f16: fp32 D, bf16 A and B; A / B MN-major
// when the flag is set (K-major otherwise).
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate),
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

__device__ __forceinline__ void tma_load(uint32_t dst, const CUtensorMap* map, int c1,
                                         int c2, uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::"
        "complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(c1), "r"(c2),
        "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 16-byte global -> shared copy; bytes past src_bytes (0 or 16) are zero.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_plain(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Barrier of the four softmax warps only.
__device__ __forceinline__ void softmax_sync() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Barrier of the softmax warps that returns how many threads passed `pred`.
__device__ __forceinline__ int softmax_sync_count(bool pred) {
    int n;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.popc.u32 %0, 1, 128, p;\n\t}"
        : "=r"(n)
        : "r"(pred ? 1u : 0u)
        : "memory");
    return n;
}

__device__ __forceinline__ void set_abort(int* flag, int* error_flags) {
    if (atomicExch(flag, 1) == 0) report(error_flags, PA_DEVERR_TIMEOUT);
}
__device__ __forceinline__ bool aborted(int* flag) {
    return *reinterpret_cast<volatile int*>(flag) != 0;
}

// One compare-exchange stage of a bitonic network over the warp's 256 keys
// (8 per lane, element i = lane * 8 + e), sorting blocks of SIZE into
// descending order at distance STRIDE: below 8 within a lane, else across.
template <int SIZE, int STRIDE>
__device__ __forceinline__ void bitonic_stage(long long (&k)[8], int lane) {
    if (STRIDE >= 8) {
        constexpr int kL = STRIDE >= 8 ? STRIDE / 8 : 1;
        const bool lower = (lane & kL) == 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const bool desc = ((lane * 8 + e) & SIZE) == 0;
            const long long other = __shfl_xor_sync(0xffffffffu, k[e], kL);
            // the lower index keeps the larger key in a descending block
            k[e] = (lower == desc) ? max(k[e], other) : min(k[e], other);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            constexpr int kS = STRIDE < 8 ? STRIDE : 1;
            if ((e ^ kS) > e) {
                const bool desc = ((lane * 8 + e) & SIZE) == 0;
                const long long a = k[e], b = k[e ^ kS];
                const bool swap = desc ? a < b : a > b;
                k[e] = swap ? b : a;
                k[e ^ kS] = swap ? a : b;
            }
        }
    }
    if constexpr (STRIDE > 1) bitonic_stage<SIZE, STRIDE / 2>(k, lane);
}

template <int SIZE>
__device__ __forceinline__ void bitonic_sizes(long long (&k)[8], int lane) {
    bitonic_stage<SIZE, SIZE / 2>(k, lane);
    if constexpr (SIZE < 256) bitonic_sizes<SIZE * 2>(k, lane);
}

// Sorts the warp's 256 keys into descending order.
__device__ __forceinline__ void warp_sort256_desc(long long (&k)[8], int lane) {
    bitonic_sizes<2>(k, lane);
}

// Lane r ends with the reduction over the warp of row r of v (v is consumed).
template <bool kMax>
__device__ __forceinline__ float transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = upper ? v[i] : v[i + o];
            const float keep = upper ? v[i + o] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
    return v[0];
}

__device__ __forceinline__ int clamp_len(const MultiRowParams& p, int s, bool report_errors) {
    int L = p.context_lens[s];
    if (L < 0 || L > p.max_context_len) {
        if (report_errors) report(p.error_flags, PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : p.max_context_len;
    }
    return L;
}

// Query count of sequence s in multi-query mode, clamped to [0, min(L, max_query_len)].
__device__ __forceinline__ int clamp_queries(const MultiRowParams& p, int s, int L,
                                             bool report_errors) {
    int k = p.query_start_loc[s + 1] - p.query_start_loc[s];
    if (k < 0 || k > L || k > p.max_query_len) {
        if (report_errors) report(p.error_flags, PA_DEVERR_QUERY_LEN);
        k = k < 0 ? 0 : min(k, min(L, p.max_query_len));
    }
    return k;
}

// Work item idx = (unit * tiles + tile) * Hkv + kv head.
struct RowItem {
    int unit;       // sequence or group; -1: nothing to do
    int tile;
    int g;
    int table_seq;  // sequence whose block table holds the shared tokens
    int range_end;  // virtual tokens [0, range_end) are streamed
    int nch;        // 128-token chunks
    int P;          // group mode: prefix length
    int shared_end; // group mode: end of the shared region
    int m0, nmem;   // group mode: first member of the tile, members
    int lane_len;   // group mode: context length of member m0 + lane (lane < nmem)
};

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

__device__ RowItem row_item(const MultiRowParams& p, int idx, bool report_errors) {
    RowItem it;
    it.unit = -1;
    const int g = idx % p.num_kv_heads;
    const int rest = idx / p.num_kv_heads;
    const int tile = rest % p.tiles;
    const int unit = rest / p.tiles;
    const int G = p.group;
    int range_end = 0, table_seq = 0;
    if (!p.shared_prefix_mode) {
        const int s = unit;
        const int L = clamp_len(p, s, report_errors);
        const int k = clamp_queries(p, s, L, report_errors && tile == 0 && g == 0);
        const int r0 = tile * kN;
        const int rows = min(kN, k * G - r0);
        if (rows <= 0) return it;
        range_end = L - k + (r0 + rows - 1) / G + 1;
        table_seq = s;
    } else {
        const int P = cascade_group_prefix(p.groups, unit, p.num_seqs, p.block_size,
                                           p.error_flags, report_errors);
        if (P == 0) return it;
        const int a = p.groups.group_start[unit];
        const int b = p.groups.group_start[unit + 1];
        const int mpt = kN / G;
        const int m0 = a + tile * mpt;
        const int m1 = min(b, m0 + mpt);
        if (m0 >= m1) return it;
        // The shared region is read through the table of the member whose
        // context covers most of it (a shorter member's table may end first;
        // ties go to the first member).  Called by a whole warp with the same
        // idx: lane m loads member m0 + m's length (at most 32 members per
        // tile), and warp reductions combine them.
        const int lane = threadIdx.x & 31;
        const bool mem = m0 + lane < m1;
        const int L = mem ? clamp_len(p, m0 + lane, report_errors) : 0;
        const int sh = mem ? min(P, L) : -1;
        int best = sh, best_s = mem ? m0 + lane : 0x7fffffff;
        int tails = mem ? round16(L - sh) : 0;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const int ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int os = __shfl_xor_sync(0xffffffffu, best_s, o);
            if (ob > best || (ob == best && os < best_s)) {
                best = ob;
                best_s = os;
            }
            tails += __shfl_xor_sync(0xffffffffu, tails, o);
        }
        const int shared_end = best;
        table_seq = best_s;
        range_end = tails > 0 ? round16(shared_end) + tails : shared_end;
        it.P = P;
        it.shared_end = shared_end;
        it.m0 = m0;
        it.nmem = m1 - m0;
        it.lane_len = L;
    }
    if (range_end <= 0) return it;
    it.unit = unit;
    it.tile = tile;
    it.g = g;
    it.table_seq = table_seq;
    it.range_end = range_end;
    it.nch = (range_end + kTok - 1) / kTok;
    return it;
}

// Work of unit u (sequence or group) for the item deal: its live row tiles
// and the weight of each of its items (128-token chunks, plus one for the
// per-item overhead).  Invalid groups have no tiles.
// Multi-query mode: tiles and weight of a sequence from its raw context
// length and query count, clamped (and reported) as clamp_len and
// clamp_queries do.
__device__ __forceinline__ void query_unit_work(const MultiRowParams& p, int L, int k,
                                                bool report_errors, int& tiles, int& w) {
    if (L < 0 || L > p.max_context_len) {
        if (report_errors) report(p.error_flags, PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : p.max_context_len;
    }
    if (k < 0 || k > L || k > p.max_query_len) {
        if (report_errors) report(p.error_flags, PA_DEVERR_QUERY_LEN);
        k = k < 0 ? 0 : min(k, min(L, p.max_query_len));
    }
    tiles = min((k * p.group + kN - 1) / kN, p.tiles);
    w = (L + kTok - 1) / kTok + 1;
}

// Group mode also returns, for a one-tile group, its item's exact chunk
// count (as row_item computes it), else 0.
__device__ __forceinline__ void unit_work(const MultiRowParams& p, int u,
                                          bool report_errors, int& tiles, int& w, int& nch) {
    nch = 0;
    if (!p.shared_prefix_mode) {
        const int L = clamp_len(p, u, report_errors);
        const int k = clamp_queries(p, u, L, report_errors);
        tiles = (k * p.group + kN - 1) / kN;
        w = (L + kTok - 1) / kTok + 1;
    } else {
        const int P = cascade_group_prefix(p.groups, u, p.num_seqs, p.block_size,
                                           p.error_flags, report_errors);
        const int a = p.groups.group_start[u];
        const int members = p.groups.group_start[u + 1] - a;
        const int mpt = kN / p.group;
        tiles = P > 0 ? (members + mpt - 1) / mpt : 0;
        long long tails = 0;
        int shared_end = 0;
        if (P > 0)
            for (int s0 = a; s0 < a + members; s0 += 8) {  // 8 loads in flight
                int Ls[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    Ls[e] = s0 + e < a + members ? clamp_len(p, s0 + e, report_errors) : -1;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (Ls[e] >= 0) {
                        tails += round16(Ls[e] - min(P, Ls[e]));
                        shared_end = max(shared_end, min(P, Ls[e]));
                    }
            }
        const long long per_tile = tiles > 0 ? tails / tiles : 0;
        w = (int)((P + per_tile + kTok - 1) / kTok) + 1;
        if (tiles == 1) {
            const long long range_end =
                tails > 0 ? round16(shared_end) + tails : (long long)shared_end;
            nch = (int)((range_end + kTok - 1) / kTok);
        }
    }
    tiles = min(tiles, p.tiles);
}

// Row r of a live item: last visible token (lim) and the q / out row index
// (-1 for a row that does not exist).
__device__ void row_of(const MultiRowParams& p, const RowItem& it, int r, int& lim,
                       long long& row) {
    lim = -1;
    row = -1;
    const int G = p.group;
    const int Hq = p.num_heads;
    if (!p.shared_prefix_mode) {
        const int s = it.unit;
        const int L = clamp_len(p, s, false);
        const int k = clamp_queries(p, s, L, false);
        const int R = it.tile * kN + r;
        if (R >= k * G) return;
        const int j = R / G;
        lim = L - k + j;
        row = (long long)(p.query_start_loc[s] + j) * Hq + it.g * G + R % G;
    } else {
        // Called by the whole warp, lane = r: member m = r / G's length is
        // in lane m of it.lane_len.
        const int mpt = kN / G;
        const int m = r / G;
        const int Lm = __shfl_sync(0xffffffffu, it.lane_len, m < 32 ? m : 0);
        if (m >= mpt || m >= it.nmem) return;
        const int s = it.m0 + m;
        lim = min(it.P, Lm) - 1;
        row = (long long)s * Hq + it.g * G + r % G;
    }
}

// Split deal of the shared-prefix group pass.  Per kv head the items (one
// per group, one tile each) lie end to end on an axis in group order: item
// u takes positions [a, a + n + 1), the first for its fixed cost, then one
// per 128-token chunk (chunk c at a + 1 + c).  CTA j of the head's `per`
// owns positions [B(j), B(j + 1)), B(j) = floor(j T / per), T the axis
// length, and attends the chunks whose positions it owns: a piece of an item
// is a run of chunks with one owner.  The piece at an item's first chunk
// writes its partial to slot u; a piece that starts at chunk c >= 1 does so
// only where a CTA's range starts (B(j) = a + 1 + c), and takes slot
// units + j.
// The deal keeps (T + 1) * per within int, so these products do not overflow.
__device__ __forceinline__ int axis_bound(int T, int per, int j) { return j * T / per; }

// Calls f(j) for every CTA j whose range starts inside item (a, n) at
// chunk 1 .. n - 1 (each such piece's slot is units + j); CTAs with empty
// ranges own nothing and are skipped.
template <typename F>
__device__ __forceinline__ void for_each_inner_piece(int a, int n, int T, int per, F&& f) {
    if (n <= 1 || T <= 0) return;
    // B(j) in [a + 2, a + n].
    int jlo = ((a + 2) * per + T - 1) / T;
    int jhi = ((a + n + 1) * per + T - 1) / T - 1;
    if (jlo < 1) jlo = 1;
    if (jhi > per - 1) jhi = per - 1;
    for (int j = jlo; j <= jhi; ++j)
        if (axis_bound(T, per, j + 1) > axis_bound(T, per, j)) f(j);
}

template <int BS>
__global__ void __launch_bounds__(kThreads, 1)
paged_multi_row_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const MultiRowParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* k_full = bars;
    uint64_t* k_empty = k_full + kKStages;
    uint64_t* v_full = k_empty + kKStages;
    uint64_t* v_empty = v_full + kVStages;
    uint64_t* s_full = v_empty + kVStages;
    uint64_t* s_free = s_full + 2;
    uint64_t* p_full = s_free + 2;
    uint64_t* pv_done = p_full + 2;
    uint64_t* o_full = pv_done + 2;
    uint64_t* o_empty = o_full + 2;
    uint64_t* q_empty = o_empty + 2;
    uint64_t* item_ready = q_empty + 2;
    uint64_t* slot_free = item_ready + kSlots;
    uint64_t* drain = slot_free + kSlots;
    uint64_t* item_meta = drain + 1;  // the slot's fields (producers); item_ready adds Q
    uint64_t* item_refs = item_meta + kSlots;  // and the rows' references (softmax)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
    int* abort_flag = reinterpret_cast<int*>(smem + kBarOff + kNumBars * 8 + 4);
    float* cmax = reinterpret_cast<float*>(smem + kCmaxOff);
    ItemSlot* slots = reinterpret_cast<ItemSlot*>(smem + kSlotOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) report(p.error_flags, PA_DEVERR_INTERNAL);
        return;
    }
    pdl_wait();
    pdl_launch_dependents();

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
            mbar_init(&s_free[i], 128);
            mbar_init(&p_full[i], 128);
            mbar_init(&pv_done[i], 1);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_empty[i], 128);
            mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&item_ready[i], 32);
            mbar_init(&item_meta[i], 32);
            mbar_init(&item_refs[i], 32);
            mbar_init(&slot_free[i], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 6) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t pol = l2_policy_evict_first();

    if (warp == 7) {
        // -------------------------------------------------------- scheduler
        int live = 0;
        // A split item's piece: chunks [c0, c1) of the item at position a
        // of an axis of length T (see the split deal); slot -1 for the whole.
        struct Piece {
            int c0, c1, slot, n, a, T;
        };
        // Publish item idx (idx < 0: the end marker), whole or one piece of
        // it; false on abort.
        auto publish = [&](int idx, const Piece& pc) -> bool {
            const bool end = idx < 0;
            RowItem it;
            it.unit = -1;
            if (!end) {
                it = row_item(p, idx, false);
                if (it.unit < 0) return true;
            }
            if (!end && pc.slot >= 0 &&
                (pc.n != it.nch || pc.c0 < 0 || pc.c1 <= pc.c0 || pc.c1 > it.nch)) {
                if (lane == 0) report(p.error_flags, PA_DEVERR_INTERNAL);
                return true;
            }
            const int s = live % kSlots;
            bool good = true;
            // The slot's previous item has been written out.
            if (lane == 0 && live >= kSlots)
                good = wait_bar(&slot_free[s], ((live / kSlots) - 1) & 1);
            // The Q buffer's previous item (live - 2) has had all its S products.
            if (good && lane == 0 && !end && live >= 2)
                good = wait_bar(&q_empty[live & 1], ((live - 2) >> 1) & 1);
            if (__shfl_sync(0xffffffffu, good ? 1 : 0, 0) == 0) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                return false;
            }
            ItemSlot& S = slots[s];
            if (end) {
                if (lane == 0) S.nch = -1;
                mbar_arrive_plain(&item_meta[s]);
                mbar_arrive_plain(&item_ready[s]);
                mbar_arrive_plain(&item_refs[s]);
                return true;
            }
            int lim;
            long long row;
            row_of(p, it, lane, lim, row);
            S.lim[lane] = lim;
            S.row[lane] = row;
            int ml = row >= 0 ? lim : 0x7fffffff;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) ml = min(ml, __shfl_xor_sync(0xffffffffu, ml, o));
            // Group mode: member `lane`'s private tail on the virtual axis
            // (after the shared region, each tail padded to 16 tokens), and
            // every row's own tail interval.
            const int shared_r16 = p.shared_prefix_mode ? round16(it.shared_end)
                                                        : round16(it.range_end);
            int mv = 0, mt = 0, mpad = 0, mseq = -1;
            if (p.shared_prefix_mode && lane < it.nmem) {
                mseq = it.m0 + lane;
                const int L = it.lane_len;
                mt = L - min(it.P, L);
                mpad = round16(mt);
            }
            int incl = mpad;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            mv = shared_r16 + incl - mpad;
            // Member lane's rows are lane * G .. lane * G + G - 1 (those that exist).
            const uint32_t live_rows = __ballot_sync(0xffffffffu, row >= 0);
            const int G = p.group;
            S.mem_seq[lane] = mseq;
            S.mem_v[lane] = mv;
            S.mem_vend[lane] = mv + mpad;
            S.mem_tend[lane] = mv + mt;
            S.mem_rows[lane] = (p.shared_prefix_mode && lane < it.nmem && lane * G < 32)
                                   ? (((1u << G) - 1u) << (lane * G)) & live_rows
                                   : 0u;
            const int my_m = row >= 0 && p.shared_prefix_mode ? lane / G : 0;
            const int t_lo = __shfl_sync(0xffffffffu, mv, my_m);
            const int t_len = __shfl_sync(0xffffffffu, mt, my_m);
            const int tail_lo = row >= 0 && p.shared_prefix_mode ? t_lo : 0;
            const int tail_hi = row >= 0 && p.shared_prefix_mode ? t_lo + t_len : 0;
            // This piece's chunks.  The deal took a split item's count from
            // the same lengths; a piece that does not fit its item is an
            // internal error and is not streamed.
            const bool split = pc.slot >= 0;
            const int c0 = split ? pc.c0 : 0;
            const int c1 = split ? pc.c1 : it.nch;
            // Row lane's first visible token in the piece: the piece's first
            // token if the row sees it (shared region, or every token up to
            // its limit in multi-query mode), else the first token of its own
            // tail inside the piece.
            int first = -1;
            if (row >= 0) {
                const int t0 = c0 * kTok;
                if (t0 <= lim) {
                    first = t0;
                } else if (tail_hi > tail_lo) {
                    const int f = max(t0, tail_lo);
                    if (f < tail_hi && f < c1 * kTok) first = f;
                }
            }
            // Row lane's reference is its logit at that token: the token's
            // block id (the shared region from the group's table, a tail from
            // its member's, as the producers map it) is loaded now and used
            // after the Q copy is under way.
            const int m_seq = __shfl_sync(0xffffffffu, mseq, my_m);
            int ref_id = 0, ref_tok = 0;
            if (first >= 0) {
                const bool in_shared = first < shared_r16;
                const int seq = in_shared ? it.table_seq : m_seq;
                ref_tok = in_shared ? first : it.P + (first - t_lo);
                ref_id = p.block_tables[(int64_t)seq * p.max_blocks_per_seq + ref_tok / BS];
            }
            if (lane == 0) {
                S.table_seq = it.table_seq;
                S.g = it.g;
                S.range_end = it.range_end;
                S.nch = c1;
                S.c0 = c0;
                S.piece = split ? pc.slot : -1;
                S.unit = it.unit;
                S.item_n = split ? pc.n : it.nch;  // the deal's count (pieces)
                S.item_a = pc.a;
                S.axis_len = pc.T;
                S.live_rows = live_rows;
                S.min_lim = ml;
                S.nmem = p.shared_prefix_mode ? it.nmem : 0;
                S.shared_r16 = shared_r16;
                S.P = p.shared_prefix_mode ? it.P : 0;
                // The producers' first block-table read, on its way to L2.
                asm volatile("prefetch.global.L2 [%0];" ::"l"(
                    p.block_tables + (int64_t)it.table_seq * p.max_blocks_per_seq +
                    (c0 * kTok) / BS));
            }
            // The producers need the fields only; the MMA warp also the Q rows.
            mbar_arrive_plain(&item_meta[s]);
            // Q^T row `lane` (K-major, 128-byte swizzle; zeros for a missing row).
            const uint32_t qb = smem_u32(smem + kQOff + (live & 1) * kQBytes);
            const unsigned char* src =
                reinterpret_cast<const unsigned char*>(p.q + (row < 0 ? 0 : row) * kD);
            const int nbytes = row < 0 ? 0 : 16;
#pragma unroll
            for (int c16 = 0; c16 < 16; ++c16)
                cp_async_16(qb + (c16 >> 3) * kQHalf + lane * 128 +
                                (((c16 & 7) ^ (lane & 7)) << 4),
                            src + c16 * 16, nbytes);
            const uint16_t* krow = nullptr;
            if (first >= 0) {
                if (ref_id < 0 || ref_id >= p.num_blocks) {
                    report(p.error_flags, PA_DEVERR_BLOCK_ID);
                    ref_id = 0;
                }
                krow = p.k_cache +
                       ((int64_t)(ref_id * BS + ref_tok % BS) * p.num_kv_heads + it.g) * kD;
            }
            cp_async_wait_all();
            fence_proxy_async_smem();
            mbar_arrive_plain(&item_ready[s]);
            // The reference: q . k in fp32 (bf16 products are exact), in the
            // softmax's log2 units.  Any value near the row's logits serves
            // (it only shifts the exponent; the softmax's growth check covers
            // a row whose logits rise far above it); the token's own weight
            // is then ~1, so the row's sum never underflows.
            float ref = 0.f;
            if (krow != nullptr) {
                const unsigned char* qrow = smem + kQOff + (live & 1) * kQBytes + lane * 128;
                float acc = 0.f;
#pragma unroll 4
                for (int c16 = 0; c16 < 16; ++c16) {
                    const uint4 qv = *reinterpret_cast<const uint4*>(
                        qrow + (c16 >> 3) * kQHalf + (((c16 & 7) ^ (lane & 7)) << 4));
                    const uint4 kv = __ldg(reinterpret_cast<const uint4*>(krow + c16 * 8));
                    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
                    const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc = fmaf(__uint_as_float(qw[e] << 16), __uint_as_float(kw[e] << 16), acc);
                        acc = fmaf(__uint_as_float(qw[e] & 0xffff0000u),
                                   __uint_as_float(kw[e] & 0xffff0000u), acc);
                    }
                }
                ref = acc * p.scale_log2;
                if (!(ref > -INFINITY)) ref = 0.f;  // an overflowed or NaN product
            }
            S.ref[lane] = ref;
            mbar_arrive_plain(&item_refs[s]);
            ++live;
            return true;
        };
        const Piece kWhole = {0, 0, -1, 0, 0, 0};

        // Deal by work.  CTA b serves kv head g = b % Hkv as the j-th of the
        // head's per_head CTAs.  The head's items are ordered (unit, tile);
        // tile t of unit u starts at position start(u) + t * w(u) of the
        // head's total T and belongs to the CTA whose share
        // [T*j/per_head, T*(j+1)/per_head) holds that start, so every item
        // has exactly one CTA.
        // Unit weights are gathered kUnitRounds * 32 units at a time (lane l
        // takes units base + 32k + l) so that their loads are in flight
        // together; with at most that many units the second pass reuses them.
        const int Hkv = p.num_kv_heads;
        const int g = blockIdx.x % Hkv;
        const int j = blockIdx.x / Hkv;
        const int per_head = gridDim.x / Hkv;
        constexpr int kUnitRounds = 8;
        int tl[kUnitRounds], w[kUnitRounds];
        int nc[kUnitRounds];  // group mode, one-tile groups: exact chunk counts
        auto gather = [&](int base, bool report_errors) {
            if (!p.shared_prefix_mode) {
                // Every round's lengths first: the error reports below are
                // atomics on a flag word that may alias the inputs, so loads
                // after one could not be issued before it.
                int Lr[kUnitRounds], q0[kUnitRounds], q1[kUnitRounds];
#pragma unroll
                for (int k = 0; k < kUnitRounds; ++k) {
                    const int u = base + k * 32 + lane;
                    const bool in = u < p.num_units;
                    Lr[k] = in ? p.context_lens[u] : 0;
                    q0[k] = in ? p.query_start_loc[u] : 0;
                    q1[k] = in ? p.query_start_loc[u + 1] : 0;
                }
#pragma unroll
                for (int k = 0; k < kUnitRounds; ++k) {
                    tl[k] = 0;
                    w[k] = 0;
                    nc[k] = 0;
                    if (base + k * 32 + lane < p.num_units)
                        query_unit_work(p, Lr[k], q1[k] - q0[k], report_errors, tl[k], w[k]);
                }
                return;
            }
#pragma unroll
            for (int k = 0; k < kUnitRounds; ++k) {
                const int u = base + k * 32 + lane;
                tl[k] = 0;
                w[k] = 0;
                nc[k] = 0;
                if (u < p.num_units) unit_work(p, u, report_errors, tl[k], w[k], nc[k]);
            }
        };
        long long T = 0;
        for (int base = 0; base < p.num_units; base += kUnitRounds * 32) {
            gather(base, blockIdx.x == 0);
            long long W = 0;
#pragma unroll
            for (int k = 0; k < kUnitRounds; ++k) W += (long long)tl[k] * w[k];
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
            T += W;
        }
        const long long lo = T * j / per_head;
        const long long hi = T * (j + 1) / per_head;
        const bool kept = p.num_units <= kUnitRounds * 32;  // tl / w still hold them
        bool stopped = false;
        // Longest first when every unit is one item and all fit the warp:
        // the units sorted by weight go to the head's CTAs in snake order
        // (0..n-1, then n-1..0, ...), pairing long items with short ones.
        bool one_tile = true;
#pragma unroll
        for (int k = 0; k < kUnitRounds; ++k) one_tile = one_tile && tl[k] <= 1;
        const bool lpt = kept && __all_sync(0xffffffffu, one_tile);
        int max_weight = 0;  // of the units with work
#pragma unroll
        for (int k = 0; k < kUnitRounds; ++k) max_weight = max(max_weight, tl[k] > 0 ? w[k] : 0);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
            max_weight = max(max_weight, __shfl_xor_sync(0xffffffffu, max_weight, o));
        // Split deal (group mode with a piece region, every group one item):
        // the head's items on the position axis described above
        // for_each_inner_piece, in group order; this CTA attends the chunks
        // whose positions it owns.
        // Split only when one item alone exceeds 1.5 times a CTA's even
        // share: whole items dealt longest first balance to within about one
        // item, and a piece costs its partial write and a share of the
        // merge.
        long long Tl = 0;  // the split deal's axis length
        int wmax = 0;      // its longest item
#pragma unroll
        for (int k = 0; k < kUnitRounds; ++k) {
            Tl += nc[k] > 0 ? nc[k] + 1 : 0;
            wmax = max(wmax, nc[k] > 0 ? nc[k] + 1 : 0);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            Tl += __shfl_xor_sync(0xffffffffu, Tl, o);
            wmax = max(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
        }
        const bool split_deal = lpt && p.shared_prefix_mode && p.piece_o != nullptr &&
                                (long long)p.num_units + per_head <= p.piece_slots &&
                                (Tl + 1) * per_head <= 0x7fffffffLL &&
                                2LL * wmax * per_head > 3LL * Tl;
        if (split_deal) {
            const int Ta = (int)Tl;
            const int A = axis_bound(Ta, per_head, j);
            const int Bd = axis_bound(Ta, per_head, j + 1);
            int run = 0;  // first position of this round's units
            for (int k = 0; k < kUnitRounds && !stopped && run < Bd; ++k) {
                int n = 0;
#pragma unroll
                for (int e = 0; e < kUnitRounds; ++e)
                    if (e == k) n = nc[e];
                const int wgt = n > 0 ? n + 1 : 0;
                int incl = wgt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                const int a = run + incl - wgt;
                const int c0 = min(max(A - a - 1, 0), n);
                const int c1 = min(max(Bd - a - 1, 0), n);
                unsigned todo = __ballot_sync(0xffffffffu, n > 0 && c1 > c0);
                while (todo != 0 && !stopped) {
                    const int i = __ffs(todo) - 1;
                    todo &= todo - 1;
                    Piece pc;
                    pc.c0 = __shfl_sync(0xffffffffu, c0, i);
                    pc.c1 = __shfl_sync(0xffffffffu, c1, i);
                    pc.n = __shfl_sync(0xffffffffu, n, i);
                    pc.a = __shfl_sync(0xffffffffu, a, i);
                    pc.T = Ta;
                    const int u = k * 32 + i;
                    pc.slot = (pc.c0 == 0 && pc.c1 == pc.n) ? -1
                              : pc.c0 == 0                  ? u
                                                            : p.num_units + j;
                    if (!publish((u * p.tiles) * Hkv + g, pc)) stopped = true;
                }
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
        } else if (lpt && p.num_units <= 32) {
            // One key per lane (unit = lane): a 15-stage bitonic sort across
            // the warp, descending; the sorted key at position pos is in
            // lane pos.
            long long k1 = (lane < p.num_units && tl[0] > 0)
                               ? ((long long)w[0] << 32) | (long long)(0xFFFFFFFFu - (uint32_t)lane)
                               : -1;
#pragma unroll
            for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
                for (int stride = size >> 1; stride >= 1; stride >>= 1) {
                    const long long other = __shfl_xor_sync(0xffffffffu, k1, stride);
                    const bool desc = (lane & size) == 0;
                    const bool lower = (lane & stride) == 0;
                    k1 = (lower == desc) ? max(k1, other) : min(k1, other);
                }
            }
            const int live_units = __popc(__ballot_sync(0xffffffffu, k1 >= 0));
            for (int r = 0; !stopped; ++r) {
                const int pos = r * per_head + ((r & 1) ? per_head - 1 - j : j);
                if (pos >= live_units) break;
                const long long kk = __shfl_sync(0xffffffffu, k1, pos);
                const int u = (int)(0xFFFFFFFFu - (uint32_t)(kk & 0xFFFFFFFFll));
                if (!publish((u * p.tiles) * Hkv + g, kWhole)) stopped = true;
            }
        } else if (lpt && max_weight <= kCountSortMaxWeight) {
            // Counting sort by weight, heavier first and lower unit first on
            // ties (the bitonic order below), in the P buffers, which are
            // idle until the first item is published: a histogram of the
            // weights, its descending prefix as start positions, then the
            // units placed in unit order.  Unit u = k * 32 + lane.  Nothing
            // reads the buffers after the first publication (below).
            int* start = reinterpret_cast<int*>(smem + kPOff);      // [weight]
            int* order = start + kCountSortMaxWeight + 1;           // [position]
            for (int v = lane; v <= max_weight; v += 32) start[v] = 0;
            __syncwarp();
#pragma unroll
            for (int k = 0; k < kUnitRounds; ++k)
                if (k * 32 + lane < p.num_units && tl[k] > 0) atomicAdd(&start[w[k]], 1);
            __syncwarp();
            int live_units = 0;
            for (int top = max_weight; top >= 0; top -= 32) {
                const int v = top - lane;  // lane 0 holds the heaviest weight of the block
                const int c = v >= 0 ? start[v] : 0;
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                __syncwarp();
                if (v >= 0) start[v] = live_units + incl - c;
                live_units += __shfl_sync(0xffffffffu, incl, 31);
            }
            __syncwarp();
            const unsigned lt = (1u << lane) - 1u;
#pragma unroll
            for (int k = 0; k < kUnitRounds; ++k) {
                const bool live = k * 32 + lane < p.num_units && tl[k] > 0;
                const int key = live ? w[k] : -1;
                const unsigned same = __match_any_sync(0xffffffffu, key);
                if (live) order[start[key] + __popc(same & lt)] = k * 32 + lane;
                __syncwarp();
                if (live && (same & lt) == 0) start[key] += __popc(same);
                __syncwarp();
            }
            // This CTA's units in snake order, taken into registers before
            // the first publication: the softmax warps write P into these
            // buffers as soon as an item is out.  The CTA's r-th item
            // (r = e * 32 + lane) is position r * per_head + (r odd ?
            // per_head - 1 - j : j); at most 256 units.
            int mine[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int r = e * 32 + lane;
                const long long pos = (long long)r * per_head + ((r & 1) ? per_head - 1 - j : j);
                mine[e] = pos < live_units ? order[pos] : -1;
            }
            __syncwarp();
            for (int r = 0; r < 256 && !stopped; ++r) {
                int own = -1;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (e == (r >> 5)) own = mine[e];
                const int u = __shfl_sync(0xffffffffu, own, r & 31);
                if (u < 0) break;
                if (!publish((u * p.tiles) * Hkv + g, kWhole)) stopped = true;
            }
        } else if (lpt) {
            // Weights too large for the counting sort: bitonic sort of
            // 64-bit keys across the warp.
            long long key[8];  // weight << 32 | (~unit): heavier first, then lower unit
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int u = lane * 8 + e;  // sort element u holds unit u
                int tu = 0, wu = 0;
#pragma unroll
                for (int k = 0; k < kUnitRounds; ++k) {  // unit u sits in lane u%32, round u/32
                    const int src_t = __shfl_sync(0xffffffffu, tl[k], u & 31);
                    const int src_w = __shfl_sync(0xffffffffu, w[k], u & 31);
                    if (k == (u >> 5)) {
                        tu = src_t;
                        wu = src_w;
                    }
                }
                key[e] = (u < p.num_units && tu > 0)
                             ? ((long long)wu << 32) | (long long)(0xFFFFFFFFu - (uint32_t)u)
                             : -1;
            }
            warp_sort256_desc(key, lane);
            int live_units = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) live_units += key[e] >= 0;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) live_units += __shfl_xor_sync(0xffffffffu, live_units, o);
            for (int r = 0; !stopped; ++r) {
                const int pos = r * per_head + ((r & 1) ? per_head - 1 - j : j);
                if (pos >= live_units) break;
                long long mine = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (e == (pos & 7)) mine = key[e];
                const long long kk = __shfl_sync(0xffffffffu, mine, pos >> 3);
                const int u = (int)(0xFFFFFFFFu - (uint32_t)(kk & 0xFFFFFFFFll));
                if (!publish((u * p.tiles) * Hkv + g, kWhole)) stopped = true;
            }
        }
        long long pos = 0;  // start of the current batch of 32 units
        for (int base = 0; !lpt && base < p.num_units && pos < hi && !stopped; base += 32) {
            const int k = (base / 32) % kUnitRounds;
            if (!kept && k == 0) gather(base, false);
            int tlk = 0, wk = 0;
#pragma unroll
            for (int e = 0; e < kUnitRounds; ++e)
                if (e == k) {
                    tlk = tl[e];
                    wk = w[e];
                }
            const long long W = (long long)tlk * wk;
            long long incl = W;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const long long total = __shfl_sync(0xffffffffu, incl, 31);
            if (pos + total > lo) {
                for (int i = 0; i < 32 && base + i < p.num_units && !stopped; ++i) {
                    const long long us = pos + __shfl_sync(0xffffffffu, incl - W, i);
                    const int ti = __shfl_sync(0xffffffffu, tlk, i);
                    const int wi = __shfl_sync(0xffffffffu, wk, i);
                    if (us >= hi) break;
                    if (us + (long long)ti * wi <= lo) continue;
                    for (int t = 0; t < ti && !stopped; ++t) {
                        const long long q = us + (long long)t * wi;
                        if (q < lo || q >= hi) continue;
                        if (!publish(((base + i) * p.tiles + t) * Hkv + g, kWhole)) stopped = true;
                    }
                }
            }
            pos += total;
        }
        if (!stopped) (void)publish(-1, kWhole);
    } else if (warp == 4 || warp == 5) {
        // ------------------------------------------------ K / V producers
        const bool is_v = warp == 5;
        const int S = is_v ? kVStages : kKStages;
        uint64_t* full = is_v ? v_full : k_full;
        uint64_t* empty = is_v ? v_empty : k_empty;
        const CUtensorMap* map = is_v ? &tm_v : &tm_k;
        const uint32_t ring = smem_u32(smem + (is_v ? kVOff : kKOff));
        int n = 0;  // chunks issued by this stream
        bool ok = true;
        for (int item = 0; ok; ++item) {
            const int sl = item % kSlots;
            if (!__all_sync(0xffffffffu, wait_bar(&item_meta[sl], (item / kSlots) & 1))) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                break;
            }
            const ItemSlot& SL = slots[sl];
            const int nch = SL.nch;
            if (nch < 0) break;
            const int c0 = SL.c0;
            const int g = SL.g;
            const int range_end = SL.range_end;
            const int shared_r16 = SL.shared_r16;
            int win = -1;  // lane l: slot of 16-token piece l of chunks c..c+3
            for (int c = c0; c < nch; ++c) {
                if (((c - c0) & 3) == 0) {
                    // Virtual token v0: shared (the group's table), or a
                    // member's tail (that member's table, after the prefix).
                    const int v0 = (c * 8 + lane) * 16;
                    int seq = -1, tok = v0;
                    if (v0 < range_end) {
                        if (v0 < shared_r16) {
                            seq = SL.table_seq;
                        } else {
                            for (int m = 0; m < SL.nmem; ++m)
                                if (v0 >= SL.mem_v[m] && v0 < SL.mem_vend[m]) {
                                    seq = SL.mem_seq[m];
                                    tok = SL.P + (v0 - SL.mem_v[m]);
                                }
                        }
                    }
                    int v = -1;
                    if (seq >= 0) {
                        int id = p.block_tables[(int64_t)seq * p.max_blocks_per_seq + tok / BS];
                        if (id < 0 || id >= p.num_blocks) {
                            report(p.error_flags, PA_DEVERR_BLOCK_ID);
                            id = 0;
                        }
                        v = id * BS + tok % BS;
                    }
                    win = v;
                }
                const int stage = n % S;
                if (n >= S) {
                    bool okw = true;
                    if (lane == 0) okw = wait_bar(&empty[stage], ((n / S) - 1) & 1);
                    if (__shfl_sync(0xffffffffu, okw ? 1 : 0, 0) == 0) {
                        if (lane == 0) set_abort(abort_flag, p.error_flags);
                        ok = false;
                        break;
                    }
                }
                if (aborted(abort_flag)) {
                    ok = false;
                    break;
                }
                const int sl16 = __shfl_sync(0xffffffffu, win, ((c - c0) & 3) * 8 + (lane & 7));
                const bool mine = lane < 8 && sl16 >= 0;
                const uint32_t pieces = __popc(__ballot_sync(0xffffffffu, mine));
                if (lane == 0) mbar_arrive_expect_tx(&full[stage], pieces * 2 * 2048);
                __syncwarp();
                if (mine) {
                    const uint32_t dst = ring + stage * kStageBytes + lane * 2048;
                    tma_load(dst, map, g * 2, sl16, &full[stage], pol);
                    tma_load(dst + kHalf, map, g * 2 + 1, sl16, &full[stage], pol);
                }
                __syncwarp();
                ++n;
            }
        }
        // Copies still in flight land before the CTA may exit.
        if (lane == 0)
            for (int m = (n > S ? n - S : 0); m < n; ++m)
                (void)wait_bar(&full[m % S], (m / S) & 1);
    } else if (warp == 6) {
        // -------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc_s = instr_desc(kTok, kN, false, false);
        constexpr uint32_t idesc_pv = instr_desc(kD, 2 * kN, true, true);
        // Base descriptors, built once; each MMA adds its offset in 16-byte
        // units (stage, buffer and K slice) to the start-address field.
        // V^T: MN-major, M = d in two 64-wide swizzle columns 16 KB apart
        // (LBO), 8-token groups 1 KB apart (SBO).  [P_hi^T | P_lo^T]:
        // MN-major, N = 64 = one swizzle column.  K and Q: K-major, 8-row
        // groups 1 KB apart; a 16-wide d slice starts 32 B into the row.
        const uint64_t v_desc0 = smem_desc(smem_u32(smem + kVOff), kHalf, 1024);
        const uint64_t p_desc0 = smem_desc(smem_u32(smem + kPOff), kPBytes, 1024);
        const uint64_t k_desc0 = smem_desc(smem_u32(smem + kKOff), 16, 1024);
        const uint64_t q_desc0 = smem_desc(smem_u32(smem + kQOff), 16, 1024);
        struct Pending {
            int n, item;
            bool first, last;
        };
        Pending pend0 = {0, 0, false, false};     // PVs still to issue:
        Pending pend1 = pend0;                    // pend0 is the older
        int npend = 0;
        bool ok = true;

        auto issue_pv = [&](const Pending& pd) -> bool {
            const int vs = pd.n % kVStages;
            bool good = true;
            if (lane == 0) good = wait_bar(&v_full[vs], (pd.n / kVStages) & 1);
            if (good && lane == 0) good = wait_bar(&p_full[pd.n & 1], (pd.n >> 1) & 1);
            if (good && lane == 0 && pd.first && pd.item >= 2)
                good = wait_bar(&o_empty[pd.item & 1], ((pd.item - 2) >> 1) & 1);
            good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
            if (!good) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                return false;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint64_t vd = v_desc0 + (uint64_t)((vs * kStageBytes) >> 4);
                const uint64_t pdesc = p_desc0 + (uint64_t)(((pd.n & 1) * kPBytes) >> 4);
                const uint32_t d_tmem = tmem + kTmemO + (pd.item & 1) * 2 * kN;
#pragma unroll
                for (int kt = 0; kt < kTok / 16; ++kt)
                    mma_ss(d_tmem, vd + (uint64_t)((kt * 2048) >> 4),
                           pdesc + (uint64_t)((kt * 2048) >> 4), idesc_pv,
                           (pd.first && kt == 0) ? 0u : 1u);
                mma_commit(&v_empty[vs]);
                mma_commit(&pv_done[pd.n & 1]);
                if (pd.last) mma_commit(&o_full[pd.item & 1]);
            }
            __syncwarp();
            return true;
        };

        int n = 0;
        for (int item = 0; ok; ++item) {
            const int sl = item % kSlots;
            // Also covers the item's Q rows, copied before publication.
            if (!__all_sync(0xffffffffu, wait_bar(&item_ready[sl], (item / kSlots) & 1))) {
                if (lane == 0) set_abort(abort_flag, p.error_flags);
                ok = false;
                break;
            }
            const int nch = slots[sl].nch;
            if (nch < 0) break;
            const int c0 = slots[sl].c0;
            const uint64_t qd = q_desc0 + (uint64_t)(((item & 1) * kQBytes) >> 4);
            for (int c = c0; c < nch; ++c, ++n) {
                bool good = true;
                if (lane == 0) {
                    good = wait_bar(&k_full[n % kKStages], (n / kKStages) & 1);
                    // S buffer n%2 held S(n-2): the softmax has loaded it.
                    if (good && n >= 2) good = wait_bar(&s_free[n & 1], ((n - 2) >> 1) & 1);
                }
                good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
                if (!good || aborted(abort_flag)) {
                    if (lane == 0) set_abort(abort_flag, p.error_flags);
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t kd =
                        k_desc0 + (uint64_t)(((n % kKStages) * kStageBytes) >> 4);
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t k_off = ((ks >> 2) * kHalf + (ks & 3) * 32) >> 4;
                        const uint32_t q_off = ((ks >> 2) * kQHalf + (ks & 3) * 32) >> 4;
                        mma_ss(tmem + (n & 1) * 32, kd + k_off, qd + q_off, idesc_s,
                               ks > 0 ? 1u : 0u);
                    }
                    mma_commit(&s_full[n & 1]);
                    mma_commit(&k_empty[n % kKStages]);
                    if (c == nch - 1) mma_commit(&q_empty[item & 1]);
                }
                __syncwarp();
                if (npend == 2) {
                    if (!issue_pv(pend0)) {
                        ok = false;
                        break;
                    }
                    pend0 = pend1;
                    npend = 1;
                }
                Pending pn;
                pn.n = n;
                pn.item = item;
                pn.first = c == c0;
                pn.last = c == nch - 1;
                if (npend == 0) pend0 = pn; else pend1 = pn;
                ++npend;
            }
        }
        if (ok && npend >= 1) ok = issue_pv(pend0);
        if (ok && npend == 2) ok = issue_pv(pend1);
        if (lane == 0) {
            mma_commit(drain);               // everything issued so far
            (void)wait_bar(drain, 0);        // drained before TMEM goes away
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax, epilogue
        const int tid = threadIdx.x;             // 0..127: token of the chunk / d
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float sl2 = p.scale_log2;
        bool fail = false;  // a bounded wait of this thread gave up
        bool stop = false;  // all four warps agreed to stop

        // Row sums of the item in slot sl from the four warps' partials.
        auto finish_sums = [&](int sl) {
            if (warp == 0) {
                ItemSlot& S = slots[sl];
                const float4 v = *reinterpret_cast<const float4*>(S.red_l[lane]);
                const float l = (v.x + v.y) + (v.z + v.w);
                S.inv_l[lane] = l > 0.f ? 1.f / l : 0.f;
                S.l_fin[lane] = l;
            }
        };
        // Merge of a split item's pieces into its output rows (thread = d),
        // by the piece that arrived last: per row, the pieces' normalised O
        // weighted by l_i 2^(m_i - m) / sum_j l_j 2^(m_j - m), m the largest
        // reference among pieces with l > 0.  Warp 0 (lane = row) forms the
        // weights of up to four pieces at a time in cmax; then every thread
        // gathers its column of those pieces, all rows at once.  The pieces
        // were written by other CTAs of this grid: read through L2.  Called
        // by all four warps between barriers (cmax is free there).
        auto merge_pieces = [&](const ItemSlot& S) {
            const int Hkv = p.num_kv_heads;
            const int per = gridDim.x / Hkv;
            // Slot of the k-th piece: the item's own, then the inner ones.
            auto slot_of = [&](int k) {
                if (k == 0) return S.unit;
                int found = -1, i = 0;
                for_each_inner_piece(S.item_a, S.item_n, S.axis_len, per, [&](int jj) {
                    if (++i == k) found = p.num_units + jj;
                });
                return found;
            };
            int npieces = 1;
            for_each_inner_piece(S.item_a, S.item_n, S.axis_len, per, [&](int) { ++npieces; });
            const float2* ml = reinterpret_cast<const float2*>(p.piece_ml);
            // Row totals (warp 0): largest reference and weight sum.
            float M = -INFINITY, Lsum = 0.f;
            if (warp == 0) {
                for (int k = 0; k < npieces; ++k) {
                    const float2 v = __ldcg(ml + ((size_t)slot_of(k) * Hkv + S.g) * kN + lane);
                    if (!(v.y > 0.f)) continue;
                    if (v.x > M) {
                        Lsum *= exp2f(M - v.x);
                        M = v.x;
                    }
                    Lsum += v.y * exp2f(v.x - M);
                }
            }
            float acc[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) acc[r] = 0.f;
            for (int k0 = 0; k0 < npieces; k0 += 4) {
                const int kn = min(4, npieces - k0);
                if (warp == 0) {
                    for (int q = 0; q < 4; ++q) {
                        float w = 0.f;
                        if (q < kn) {
                            const float2 v =
                                __ldcg(ml + ((size_t)slot_of(k0 + q) * Hkv + S.g) * kN + lane);
                            w = (v.y > 0.f && Lsum > 0.f) ? v.y * exp2f(v.x - M) / Lsum : 0.f;
                        }
                        cmax[q * 32 + lane] = w;
                    }
                }
                softmax_sync();
                for (int q = 0; q < kn; ++q) {
                    const float* po =
                        p.piece_o + ((size_t)slot_of(k0 + q) * Hkv + S.g) * kN * kD + tid;
                    float o[32];
#pragma unroll
                    for (int r = 0; r < 32; ++r) o[r] = __ldcg(po + (size_t)r * kD);
#pragma unroll
                    for (int r = 0; r < 32; r += 4) {
                        const float4 w4 = *reinterpret_cast<const float4*>(cmax + q * 32 + r);
                        acc[r] += w4.x * o[r];
                        acc[r + 1] += w4.y * o[r + 1];
                        acc[r + 2] += w4.z * o[r + 2];
                        acc[r + 3] += w4.w * o[r + 3];
                    }
                }
                softmax_sync();  // cmax is rewritten by the next batch
            }
#pragma unroll
            for (int r = 0; r < 32; r += 2) {
                const longlong2 rr = *reinterpret_cast<const longlong2*>(&S.row[r]);
                if (rr.x >= 0) p.out[rr.x * kD + tid] = acc[r];
                if (rr.y >= 0) p.out[rr.y * kD + tid] = acc[r + 1];
            }
        };
        // Epilogue of item i (slot sl): O^T (thread = d) / l into the output rows
        // (one 4-byte store per row and thread; rows of one warp coalesce).  A
        // piece of a split item writes its partial instead and counts itself
        // on the item's counter; the last to arrive merges the item.
        auto epilogue = [&](int i, int sl) {
            ItemSlot& S = slots[sl];
            const int ob = i & 1;
            const bool piece = S.piece >= 0;
            bool okw = __all_sync(0xffffffffu, wait_bar(&o_full[ob], (i >> 1) & 1));
            // A piece's epilogue has barriers: the four warps agree first.
            if (piece) okw = softmax_sync_count(!okw) == 0;
            if (!okw) {
                fail = true;
                return;
            }
            tc_fence_after();
            uint32_t o[32], olo[32];
            tmem_ld32(tmem + kTmemO + ob * 2 * kN + lane_off, o);
            tmem_ld32(tmem + kTmemO + ob * 2 * kN + kN + lane_off, olo);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive_plain(&o_empty[ob]);
            if (!piece) {
#pragma unroll
                for (int r = 0; r < 32; r += 4) {
                    const float4 iv = *reinterpret_cast<const float4*>(&S.inv_l[r]);
                    const longlong2 ra = *reinterpret_cast<const longlong2*>(&S.row[r]);
                    const longlong2 rb = *reinterpret_cast<const longlong2*>(&S.row[r + 2]);
                    const float inv[4] = {iv.x, iv.y, iv.z, iv.w};
                    const long long row[4] = {ra.x, ra.y, rb.x, rb.y};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (row[e] >= 0)
                            p.out[row[e] * kD + tid] =
                                (__uint_as_float(o[r + e]) + __uint_as_float(olo[r + e])) *
                                inv[e];
                }
                mbar_arrive_plain(&slot_free[sl]);
                return;
            }
            const int Hkv = p.num_kv_heads;
            const size_t base = ((size_t)S.piece * Hkv + S.g) * kN;
            float* po = p.piece_o + base * kD + tid;
#pragma unroll
            for (int r = 0; r < 32; r += 4) {
                const float4 iv = *reinterpret_cast<const float4*>(&S.inv_l[r]);
                const float inv[4] = {iv.x, iv.y, iv.z, iv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    po[(size_t)(r + e) * kD] =
                        (__uint_as_float(o[r + e]) + __uint_as_float(olo[r + e])) * inv[e];
            }
            if (tid < 32)
                reinterpret_cast<float2*>(p.piece_ml)[base + tid] =
                    make_float2(S.m_fin[tid], S.l_fin[tid]);
            // Release the partial, count it, and acquire the others' if this
            // piece is the last: the barrier orders every thread's stores
            // before thread 0's fences and atomic.
            softmax_sync();
            if (tid == 0) {
                __threadfence();
                S.arrived = atomicAdd(&p.piece_count[(size_t)S.unit * Hkv + S.g], 1);
                __threadfence();
            }
            softmax_sync();
            int pieces = 1;
            for_each_inner_piece(S.item_a, S.item_n, S.axis_len, gridDim.x / Hkv,
                                 [&](int) { ++pieces; });
            if (S.arrived == pieces - 1) merge_pieces(S);
            mbar_arrive_plain(&slot_free[sl]);
        };

        // Reference and partial sum per row; the reference starts as the
        // row's logit at its first visible token of the item (the
        // scheduler's; its tokens before that are masked).
        float m_ref[32], l_part[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            m_ref[r] = 0.f;
            l_part[r] = 0.f;
        }
        int n = 0, item = 0;
        int prev = -1;  // slot of the item whose epilogue is pending
        // This token's 128-byte row of [P_hi^T | P_lo^T] (MN-major, 128-byte
        // swizzle: 16-byte chunk j of row t sits at chunk j ^ (t % 8)).
        const uint32_t p_row = (uint32_t)tid * 128;
        const uint32_t p_sw = (uint32_t)(tid & 7);

        for (;; ++item) {
            const int sl = item % kSlots;
            const bool okw = wait_bar(&item_refs[sl], (item / kSlots) & 1);
            // One barrier per item: the four warps agree on stopping, and the
            // previous item's partial sums are visible.
            const bool bad = !okw || fail || (tid == 0 && aborted(abort_flag));
            if (softmax_sync_count(bad) != 0) {
                if (tid == 0) set_abort(abort_flag, p.error_flags);
                stop = true;
                break;
            }
            ItemSlot& S = slots[sl];
            const int nch = S.nch;
            if (nch < 0) break;
            const int c0 = S.c0;
            if (prev >= 0) finish_sums(prev);
            const int min_lim = S.min_lim;
            const int ob = item & 1;
            const uint32_t live_rows = S.live_rows;
#pragma unroll
            for (int r = 0; r < 32; r += 4) {
                const float4 r4 = *reinterpret_cast<const float4*>(&S.ref[r]);
                m_ref[r] = r4.x;
                m_ref[r + 1] = r4.y;
                m_ref[r + 2] = r4.z;
                m_ref[r + 3] = r4.w;
            }

            for (int c = c0; c < nch; ++c, ++n) {
                const int sb = n & 1;
                bool ok = !fail && __all_sync(0xffffffffu, wait_bar(&s_full[sb], (n >> 1) & 1));
                float x[32];
                bool dead = false;  // no row sees this thread's token
                const int tok = c * kTok + tid;
                if (ok) {
                    tc_fence_after();
                    uint32_t raw[32];
                    tmem_ld32(tmem + sb * 32 + lane_off, raw);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive_plain(&s_free[sb]);  // S(n+2) may overwrite the buffer
#pragma unroll
                    for (int r = 0; r < 32; ++r) x[r] = __uint_as_float(raw[r]) * sl2;
                    if (c * kTok + kTok - 1 > min_lim) {
                        // The rows that see this token: every row up to the
                        // smallest limit; in the shared region (or in
                        // multi-query mode) those whose limit reaches it;
                        // past it, the rows of the one member whose tail
                        // holds it (none on a tail's padding).
                        uint32_t vis = live_rows;
                        if (tok > min_lim) {
                            if (tok < S.shared_r16) {
                                vis = 0;
#pragma unroll
                                for (int r = 0; r < 32; r += 4) {
                                    const int4 lm = *reinterpret_cast<const int4*>(&S.lim[r]);
                                    vis |= (tok <= lm.x ? 1u : 0u) << r;
                                    vis |= (tok <= lm.y ? 2u : 0u) << r;
                                    vis |= (tok <= lm.z ? 4u : 0u) << r;
                                    vis |= (tok <= lm.w ? 8u : 0u) << r;
                                }
                                vis &= live_rows;
                            } else {
                                // The last member whose tail starts at or
                                // before tok (tails rise with the member):
                                // a branch-free search over at most 32.
                                const int nm = S.nmem;
                                int lo = 0;
#pragma unroll
                                for (int step = 16; step >= 1; step >>= 1)
                                    if (lo + step < nm && S.mem_v[lo + step] <= tok) lo += step;
                                vis = (nm > 0 && S.mem_v[lo] <= tok && tok < S.mem_tend[lo])
                                          ? S.mem_rows[lo]
                                          : 0u;
                            }
                        }
#pragma unroll
                        for (int r = 0; r < 32; ++r)
                            if (!((vis >> r) & 1u)) x[r] = -INFINITY;
                        dead = vis == 0;
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < 32; ++r) x[r] = -INFINITY;
                }
                bool grow = false;
#pragma unroll
                for (int r = 0; r < 32; ++r) grow = grow || x[r] > m_ref[r] + kRescaleThreshold;
                if (lane == 0 && aborted(abort_flag)) ok = false;
                ok = __all_sync(0xffffffffu, ok);
                const bool slow = softmax_sync_count(grow || !ok) != 0;
                if (__builtin_expect(slow, 0) && softmax_sync_count(!ok) != 0) {
                    if (tid == 0) set_abort(abort_flag, p.error_flags);
                    stop = true;
                    break;
                }
                if (__builtin_expect(slow, 0)) {
                    // Exact chunk max per row, then move the references.
                    float v[32];
#pragma unroll
                    for (int r = 0; r < 32; ++r) v[r] = x[r];
                    cmax[lane * 4 + warp] = transpose_reduce<true>(v, lane);
                    softmax_sync();
                    float alpha[32];
                    bool resc = false;
#pragma unroll
                    for (int r = 0; r < 32; ++r) {
                        const float4 c4 = *reinterpret_cast<const float4*>(cmax + r * 4);
                        const float cm = fmaxf(fmaxf(c4.x, c4.y), fmaxf(c4.z, c4.w));
                        const float mn = fmaxf(m_ref[r], cm);
                        alpha[r] = exp2f(m_ref[r] - mn);
                        resc = resc || mn != m_ref[r];
                        m_ref[r] = mn;
                        l_part[r] *= alpha[r];
                    }
                    if (resc && c > c0) {
                        // O^T must be stable: the previous PV has to be done.
                        const bool okp = __all_sync(
                            0xffffffffu, wait_bar(&pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1));
                        if (okp) {
                            tc_fence_after();
#pragma unroll
                            for (int part = 0; part < 2; ++part) {
                                const uint32_t ta = tmem + kTmemO + ob * 2 * kN + part * kN + lane_off;
                                uint32_t o[32];
                                tmem_ld32(ta, o);
                                tmem_wait_ld();
#pragma unroll
                                for (int r = 0; r < 32; ++r)
                                    o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha[r]);
                                tmem_st32(ta, o);
                            }
                            tmem_wait_st();
                        } else {
                            fail = true;
                        }
                    }
                }
                // P buffer sb is free once PV(n-2) is done.
                if (n >= 2 && !__all_sync(0xffffffffu,
                                          wait_bar(&pv_done[sb], ((n - 2) >> 1) & 1)))
                    fail = true;
                // P = 2^(x - m) as bf16 plus its bf16 residual, both rounded
                // to nearest (P carries ~17 bits into PV).
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float a = exp2f(x[2 * i] - m_ref[2 * i]);
                    const float b = exp2f(x[2 * i + 1] - m_ref[2 * i + 1]);
                    l_part[2 * i] += a;
                    l_part[2 * i + 1] += b;
                    split_bf16x2(a, b, hi[i], lo[i]);
                }
                unsigned char* prow = smem + kPOff + sb * kPBytes + p_row;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t* src = j < 4 ? &hi[4 * j] : &lo[4 * (j - 4)];
                    *reinterpret_cast<uint4*>(prow + ((j ^ p_sw) << 4)) =
                        make_uint4(src[0], src[1], src[2], src[3]);
                }
                if (dead) {
                    // No row sees this token: its V row may hold anything
                    // (another block's rows, unwritten memory); P is 0 there,
                    // but 0 x NaN is NaN.  Cleared once the V chunk landed,
                    // as late as possible so the wait rarely blocks.
                    const int vs = n % kVStages;
                    if (!wait_bar(&v_full[vs], (n / kVStages) & 1)) fail = true;
                    // Rows are 128 bytes apart: thread t starts at 16-byte
                    // column t % 8 so that eight lanes cover all banks.
                    unsigned char* vr = smem + kVOff + vs * kStageBytes + tid * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int col = ((j + tid) & 7) * 16;
                        *reinterpret_cast<uint4*>(vr + col) = make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4*>(vr + kHalf + col) = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive_plain(&p_full[sb]);

                // The previous item's epilogue, one chunk into this item when
                // there is one: its last PV is then done, not just issued.
                if (__builtin_expect(prev >= 0 && c - c0 == min(1, nch - c0 - 1), 0)) {
                    epilogue(item - 1, prev);
                    prev = -1;
                }
            }
            if (stop) break;
            // Item end: per-row partial sums of this warp's 32 tokens.
            {
                float v[32];
#pragma unroll
                for (int r = 0; r < 32; ++r) v[r] = l_part[r];
                S.red_l[lane][warp] = transpose_reduce<false>(v, lane);
                if (tid == 0) {
#pragma unroll
                    for (int r = 0; r < 32; ++r) S.m_fin[r] = m_ref[r];
                }
#pragma unroll
                for (int r = 0; r < 32; ++r) l_part[r] = 0.f;
            }
            prev = sl;
        }
        if (prev >= 0 && !stop) {
            softmax_sync();  // the last item's partial sums
            finish_sums(prev);
            softmax_sync();
            epilogue(item - 1, prev);
        }
        if (fail && tid == 0) set_abort(abort_flag, p.error_flags);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 6)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                   void*, const cuuint64_t*, const cuuint64_t*,
                                   const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn mr_encode_fn() {
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

// Pool [NB*bs][Hkv][D] as {64 elements, Hkv*D/64 column tiles, NB*bs slots};
// box = one 128-byte column tile of 16 slots.
bool mr_encode_map(CUtensorMap* map, const void* pool, int num_blocks, int block_size,
                   int num_kv_heads) {
    EncodeTiledFn fn = mr_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)num_kv_heads * kD / 64,
                                (cuuint64_t)num_blocks * block_size};
    const cuuint64_t strides[2] = {128, (cuuint64_t)num_kv_heads * kD * 2};
    const cuuint32_t box[3] = {64, 1, 16};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pool), dims,
              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() { return device_sm_count(); }

template <int BS>
cudaError_t mr_launch_typed(const MultiRowParams& p, cudaStream_t stream) {
    static int ready[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE)) {
        e = cudaFuncSetAttribute(paged_multi_row_kernel<BS>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
    }
    CUtensorMap tmk, tmv;
    if (!mr_encode_map(&tmk, p.k_cache, p.num_blocks, BS, p.num_kv_heads) ||
        !mr_encode_map(&tmv, p.v_cache, p.num_blocks, BS, p.num_kv_heads))
        return cudaErrorInvalidValue;
    const long long items = (long long)p.num_units * p.tiles * p.num_kv_heads;
    if (items <= 0) return cudaSuccess;
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
    // One kv head per CTA, the same number of CTAs for every head (at least
    // one per head, at most one per item).
    long long per_head = multi_row_ctas_per_head(p.num_kv_heads);
    const long long head_items = (long long)p.num_units * p.tiles;
    if (per_head > head_items) per_head = head_items;
    if (per_head < 1) per_head = 1;
    const long long grid = per_head * p.num_kv_heads;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);  // gridDim.x % num_kv_heads == 0
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, paged_multi_row_kernel<BS>, tmk, tmv, p);
    count_launch();
    return e;
}

}  // namespace

int multi_row_ctas_per_head(int num_kv_heads) {
    const int n = num_sms() / (num_kv_heads > 0 ? num_kv_heads : 1);
    return n > 0 ? n : 1;
}

cudaError_t launch_paged_multi_row(const MultiRowParams& p, cudaStream_t stream) {
    if (p.block_size == 16) return mr_launch_typed<16>(p, stream);
    if (p.block_size == 32) return mr_launch_typed<32>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
