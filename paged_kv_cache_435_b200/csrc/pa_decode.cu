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
// Kernel structure (one CTA per (kv head, KV partition, sequence)):
//  * 4 warps; warp w owns 16-token chunks w, w+4, w+8, ... of the partition
//    and runs its own ring of shared-memory stages, each guarded by an
//    mbarrier with a transaction count.  A chunk is 16 K rows + 16 V rows of
//    head_size bf16 each; every lane issues one bulk asynchronous copy
//    (cp.async.bulk, executed by the TMA unit) per row, so one warp
//    instruction puts a whole chunk in flight.  Rows land at a padded stride
//    (head_size*2 + 16 bytes) so ldmatrix reads are bank-conflict free.
//  * All G = num_heads/num_kv_heads query heads of the kv head are folded
//    into one pass: S = Q K^T and O += P V run on the bf16 tensor cores with
//    mma.m16n8k16, rows 0..7 of the 16-row M tile holding the G heads.  The
//    spare rows 8..15 carry the low-order bf16 part of P (P = P_hi + P_lo),
//    so the PV product keeps ~16 bits of P instead of bf16's 8.
//  * fp32 online softmax in the log2 domain (exp2f), per-warp running max
//    and sum; the warps merge through shared memory at the end.
//  * Contexts longer than the partition are split; each partition writes its
//    max, sum and normalised output, and pa_decode_reduce_kernel merges them.
#include <cfloat>
#include <cstdint>

#include "pa_common.cuh"
#include "pa_decode.cuh"

namespace pa {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 16;  // tokens per pipeline stage (one M/K tile)
constexpr int kMaxGroup = 8;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
    static constexpr int kRowBytes = D * 2 + 16;
    static constexpr int kStageBytes = 2 * kChunk * kRowBytes;
    static constexpr int kStagesRaw = 26112 / kStageBytes;
    static constexpr int kStages = kStagesRaw < 2 ? 2 : kStagesRaw;
    static constexpr int kBarBytes = (kWarps * kStages * 8 + 127) / 128 * 128;
    static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
    static constexpr int kMergeBytes = kWarps * kMaxGroup * (D + 2) * 4;
    static constexpr int kSmemBytes =
        kBarBytes + (kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes);
    static_assert(kWarps * kStages * 8 <= kBarBytes, "barrier area");
};

template <int D, int BS>
__global__ void __launch_bounds__(kThreads, 2)
paged_decode_kernel(const DecodeParams p) {
    using C = Cfg<D>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    unsigned char* ring = smem + C::kBarBytes;

    const int g = blockIdx.x;     // kv head
    const int part = blockIdx.y;  // KV partition
    const int s = blockIdx.z;     // sequence
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.group;
    const int Hq = p.num_heads;

    int L = p.context_lens[s];
    if (L < 0 || L > p.max_context_len) {
        if (threadIdx.x == 0 && g == 0 && part == 0)
            report(p.error_flags, PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : p.max_context_len;
    }
    const int tok0 = part * p.partition_size;
    if (L == 0) {  // empty context: zeros, written once per (seq, kv head)
        if (part == 0)
            for (int i = threadIdx.x; i < G * D; i += kThreads)
                p.out[((int64_t)s * Hq + g * G + i / D) * D + i % D] = 0.f;
        return;
    }
    if (tok0 >= L) return;  // partition past this sequence's end
    const int num_parts = (L + p.partition_size - 1) / p.partition_size;
    const int tok1 = min(L, tok0 + p.partition_size);
    const int nchunks = (tok1 - tok0 + kChunk - 1) / kChunk;
    const int my_n = nchunks > warp ? (nchunks - warp + kWarps - 1) / kWarps : 0;

    uint64_t* my_bars = bars + warp * C::kStages;
    unsigned char* my_ring = ring + warp * C::kStages * C::kStageBytes;
    if (lane == 0) {
        for (int i = 0; i < C::kStages; ++i) mbar_init(&my_bars[i], 1);
        mbar_init_fence();
    }
    __syncwarp();

    // Q fragments (A operand, rows = heads of the group, rows >= G zero).
    const int qr = lane >> 2;       // fragment row owned by this lane
    const int qc = (lane & 3) * 2;  // fragment column pair
    uint32_t qa[D / 16][2];
    {
        const bool live = qr < G;
        const uint16_t* qp = p.q + ((int64_t)s * Hq + g * G + (live ? qr : 0)) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = live ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + qc) : 0u;
            qa[ks][1] = live ? *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8 + qc) : 0u;
        }
    }

    const uint64_t pol = l2_policy_evict_first();
    const int64_t tok_stride = (int64_t)p.num_kv_heads * D;  // elements
    const uint16_t* kbase = p.k_cache + (int64_t)g * D;
    const uint16_t* vbase = p.v_cache + (int64_t)g * D;
    const int32_t* bt = p.block_tables + (int64_t)s * p.max_blocks_per_seq;

    // Lane j keeps the physical block of this warp's chunk (32*k + j).
    int ids = 0;
    auto load_ids = [&](int j0) {
        const int j = j0 + lane;
        int id = 0;
        if (j < my_n) {
            const int ctok = tok0 + (warp + kWarps * j) * kChunk;
            id = bt[ctok / BS];
            if (id < 0 || id >= p.num_blocks) {
                report(p.error_flags, PA_DEVERR_BLOCK_ID);
                id = 0;
            }
        }
        ids = id;
    };

    // Put chunk j of this warp in flight (warp-uniform call).
    auto issue = [&](int j) {
        if ((j & 31) == 0) load_ids(j);
        const int phys = __shfl_sync(0xffffffffu, ids, j & 31);
        const int ctok = tok0 + (warp + kWarps * j) * kChunk;  // first token
        const int valid = min(kChunk, tok1 - ctok);
        const int off = ctok % BS;                             // row in block
        unsigned char* st = my_ring + (j % C::kStages) * C::kStageBytes;
        uint64_t* bar = &my_bars[j % C::kStages];
        fence_proxy_async_smem();
        if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(2 * valid * D * 2));
        __syncwarp();
        const bool is_v = lane >= kChunk;
        const int t = lane & (kChunk - 1);
        unsigned char* dst = st + lane * C::kRowBytes;
        if (t < valid) {
            const uint16_t* src = (is_v ? vbase : kbase) +
                                  ((int64_t)phys * BS + off + t) * tok_stride;
            bulk_g2s(dst, src, D * 2, bar, pol);
        } else if (is_v) {
            // Rows past the context: V must be finite (P is 0 there).
            uint4* z = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int c = 0; c < D * 2 / 16; ++c) z[c] = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
    };

    float o[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m_run = -INFINITY;  // running max of scaled logits (log2 domain)
    float l_run = 0.f;        // this lane's share of the running sum
    const float sl2 = p.scale_log2;

    const int pre = my_n < C::kStages ? my_n : C::kStages;
    for (int j = 0; j < pre; ++j) issue(j);

    int consumed = 0;
    bool aborted = false;
    for (int j = 0; j < my_n; ++j) {
        const int stage = j % C::kStages;
        const bool ok = mbar_wait_bounded(&my_bars[stage], (j / C::kStages) & 1);
        if (!__all_sync(0xffffffffu, ok)) {
            aborted = true;
            break;
        }
        consumed = j + 1;
        const int ctok = tok0 + (warp + kWarps * j) * kChunk;
        const uint32_t kaddr = smem_u32(my_ring + stage * C::kStageBytes);
        const uint32_t vaddr = kaddr + kChunk * C::kRowBytes;

        // S (16 rows x 16 tokens) = Q K^T, as two n8 tiles of tokens.
        float sacc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
            const uint32_t row = kaddr + (nt * 8 + (lane & 7)) * C::kRowBytes +
                                 (lane >> 3) * 16;
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(b0, b1, b2, b3, row + kk * 64);
                mma_bf16_16816(sacc[nt], qa[2 * kk][0], 0u, qa[2 * kk][1], 0u, b0, b1);
                mma_bf16_16816(sacc[nt], qa[2 * kk + 1][0], 0u, qa[2 * kk + 1][1], 0u, b2, b3);
            }
        }

        // Online softmax over this chunk for row qr (quad = 16 tokens).
        float sv[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int tok = ctok + nt * 8 + qc + e;
                sv[nt * 2 + e] = tok < tok1 ? sacc[nt][e] * sl2 : -INFINITY;
            }
        float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = exp2f(m_run - m_new);
        m_run = m_new;
        float pv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pv[e] = exp2f(sv[e] - m_new);
        l_run = l_run * alpha + ((pv[0] + pv[1]) + (pv[2] + pv[3]));
#pragma unroll
        for (int j2 = 0; j2 < D / 8; ++j2) {
            o[j2][0] *= alpha; o[j2][1] *= alpha;
            o[j2][2] *= alpha; o[j2][3] *= alpha;
        }

        // P as the A operand: rows 0..7 = bf16(P), rows 8..15 = bf16(P - bf16(P)).
        const float h0 = bf16_round(pv[0]), h1 = bf16_round(pv[1]);
        const float h2 = bf16_round(pv[2]), h3 = bf16_round(pv[3]);
        const uint32_t a0 = pack_bf16x2(h0, h1);
        const uint32_t a2 = pack_bf16x2(h2, h3);
        const uint32_t a1 = pack_bf16x2(pv[0] - h0, pv[1] - h1);
        const uint32_t a3 = pack_bf16x2(pv[2] - h2, pv[3] - h3);

        // O (16 x D) += P (16 x 16 tokens) V (16 tokens x D).
        const uint32_t vrow = vaddr +
                              ((lane & 7) + ((lane >> 3) & 1) * 8) * C::kRowBytes +
                              (lane >> 4) * 16;
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_trans(b0, b1, b2, b3, vrow + dp * 32);
            mma_bf16_16816(o[2 * dp], a0, a1, a2, a3, b0, b1);
            mma_bf16_16816(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
        }
        __syncwarp();
        if (j + C::kStages < my_n) issue(j + C::kStages);
    }

    if (aborted) {
        // Report, then drain this warp's copies still in flight (bounded)
        // before the CTA may exit or reuse the ring.
        if (lane == 0) report(p.error_flags, PA_DEVERR_TIMEOUT);
        const int issued = min(my_n, consumed + C::kStages);
        for (int j = consumed; j < issued; ++j)
            (void)mbar_wait_bounded(&my_bars[j % C::kStages], (j / C::kStages) & 1);
        m_run = -INFINITY;
        l_run = 0.f;
    }

    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

    // Merge the warps through shared memory (the ring is free now).
    __syncthreads();
    float* red_o = reinterpret_cast<float*>(ring);           // [warps][8][D]
    float* red_m = red_o + kWarps * kMaxGroup * D;             // [warps][8]
    float* red_l = red_m + kWarps * kMaxGroup;                 // [warps][8]
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        float* dst = red_o + (warp * kMaxGroup + qr) * D + 8 * j + qc;
        dst[0] = o[j][0] + o[j][2];
        dst[1] = o[j][1] + o[j][3];
    }
    if ((lane & 3) == 0) {
        red_m[warp * kMaxGroup + qr] = m_run;
        red_l[warp * kMaxGroup + qr] = l_run;
    }
    __syncthreads();

    for (int i = threadIdx.x; i < G * D; i += kThreads) {
        const int r = i / D;
        const int d = i - r * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w * kMaxGroup + r]);
        float acc = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float mw = red_m[w * kMaxGroup + r];
            const float sc = mw == -INFINITY ? 0.f : exp2f(mw - M);
            acc += sc * red_o[(w * kMaxGroup + r) * D + d];
            den += sc * red_l[w * kMaxGroup + r];
        }
        const int h = g * G + r;
        const float val = acc / den;
        if (num_parts == 1) {
            p.out[((int64_t)s * Hq + h) * D + d] = val;
        } else {
            const int64_t idx = ((int64_t)s * Hq + h) * p.max_partitions + part;
            p.tmp_o[idx * D + d] = val;
            if (d == 0) {
                p.tmp_m[idx] = M;
                p.tmp_l[idx] = den;
            }
        }
    }
}

// Merge of the per-partition results: out = sum_p w_p o_p / sum_p w_p with
// w_p = l_p * 2^(m_p - max_p m_p).  One CTA per (query head, sequence).
template <int D>
__global__ void __launch_bounds__(D)
paged_decode_reduce_kernel(const DecodeParams p) {
    const int h = blockIdx.x;
    const int s = blockIdx.y;
    int L = p.context_lens[s];
    L = L < 0 ? 0 : (L > p.max_context_len ? p.max_context_len : L);
    const int np = (L + p.partition_size - 1) / p.partition_size;
    if (np <= 1) return;  // written directly by the partition kernel
    const int64_t base = ((int64_t)s * p.num_heads + h) * p.max_partitions;

    __shared__ float warp_max[D / 32];
    float M = -INFINITY;
    for (int i = threadIdx.x; i < np; i += D) M = fmaxf(M, p.tmp_m[base + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = M;
    __syncthreads();
    M = warp_max[0];
#pragma unroll
    for (int w = 1; w < D / 32; ++w) M = fmaxf(M, warp_max[w]);

    const int d = threadIdx.x;
    float acc = 0.f, den = 0.f;
    for (int i = 0; i < np; ++i) {
        const float w = p.tmp_l[base + i] * exp2f(p.tmp_m[base + i] - M);
        acc += w * p.tmp_o[(base + i) * D + d];
        den += w;
    }
    p.out[((int64_t)s * p.num_heads + h) * D + d] = acc / den;
}

template <int D, int BS>
cudaError_t launch_typed(const DecodeParams& p, int num_seqs,
                         cudaStream_t stream) {
    using C = Cfg<D>;
    static int configured[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!__atomic_load_n(&configured[dev], __ATOMIC_ACQUIRE)) {
        cudaError_t e = cudaFuncSetAttribute(
            paged_decode_kernel<D, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
            C::kSmemBytes);
        if (e != cudaSuccess) return e;
        __atomic_store_n(&configured[dev], 1, __ATOMIC_RELEASE);
    }
    dim3 grid((unsigned)p.num_kv_heads, (unsigned)p.max_partitions,
              (unsigned)num_seqs);
    paged_decode_kernel<D, BS><<<grid, kThreads, C::kSmemBytes, stream>>>(p);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.max_partitions > 1) {
        dim3 rgrid((unsigned)p.num_heads, (unsigned)num_seqs);
        paged_decode_reduce_kernel<D><<<rgrid, D, 0, stream>>>(p);
        count_launch();
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace

float log2e_scale(float scale) { return scale * kLog2e; }

cudaError_t launch_paged_decode(const DecodeParams& p, int num_seqs,
                                int head_size, int block_size,
                                cudaStream_t stream) {
    if (head_size == 128 && block_size == 16) return launch_typed<128, 16>(p, num_seqs, stream);
    if (head_size == 128 && block_size == 32) return launch_typed<128, 32>(p, num_seqs, stream);
    if (head_size == 64 && block_size == 16) return launch_typed<64, 16>(p, num_seqs, stream);
    if (head_size == 64 && block_size == 32) return launch_typed<64, 32>(p, num_seqs, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
