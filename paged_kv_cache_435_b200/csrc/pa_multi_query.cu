// Multi-query paged attention for sm_100a: k new query tokens per sequence,
// causal within the chunk.  This is the attention of a chunked-prefill chunk
// and of speculative-decoding verification, where the large model checks all
// k proposed tokens in one pass ("vLLM: Anatomy and Mechanisms of
// High-Throughput LLM Inference", "Chunked Prefill" and "Speculative
// Decoding"; "Inside vLLM: Anatomy of a High-Throughput LLM Inference
// System", "Scheduler": the tokens per step are not always 1).
//
// Sequence s has L cached tokens (the k new ones included, already written
// by reshape_and_cache); query token j sits at position L-k+j and sees
// tokens 0..L-k+j.  Rows of the work are (query token, query head) pairs of
// one kv head: row r = j*G + gi.
//
// CTA = (kv head, 16*W-row tile, sequence), W in {1,2,4} consumer warps plus
// one producer warp.  The producer streams 16-token K/V chunks of the tile's
// causal range through a CTA-shared ring (TMA tensor tiles with 128-byte
// swizzle, full/empty mbarriers); each consumer warp owns a 16-row M tile:
// S = Q K^T and O += P V on bf16 mma.m16n8k16 with fp32 online softmax.  P
// enters the PV product as bf16(P) plus bf16(P - bf16(P)) in two passes, so
// it keeps ~16 bits.  The last chunk's rows past the tile's range are masked
// in registers (S to -inf, the V fragments to zero).
#include <cuda.h>

#include <cstdint>
#include <mutex>
#include <utility>

#include "pa_common.cuh"
#include "pa_multi_query.cuh"

namespace pa {
namespace {

constexpr int kChunk = 16;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct MQCfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kHalfBytes = kChunk * 128;
    static constexpr int kKVBytes = kHalves * kHalfBytes;
    static constexpr int kStageBytes = 2 * kKVBytes;
    static constexpr int kStages = D == 128 ? 8 : 12;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kBarOff = kRingBytes;
    static constexpr int kSmemBytes = kRingBytes + 2 * kStages * 8 + 16;
};

__device__ __forceinline__ void mq_tma_load(uint32_t dst, const CUtensorMap* map,
                                            int c0, int c1, int c2,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::"
        "complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2),
        "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Keep the bf16 halves of a B fragment whose token index is below `valid`.
__device__ __forceinline__ uint32_t keep_tokens(uint32_t b, int tok, int valid) {
    const uint32_t lo = tok < valid ? 0x0000ffffu : 0u;
    const uint32_t hi = tok + 1 < valid ? 0xffff0000u : 0u;
    return b & (lo | hi);
}

template <int D, int BS, int W>
__global__ void __launch_bounds__((W + 1) * 32)
paged_multi_query_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const MultiQueryParams p) {
    using C = MQCfg<D>;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* empty = full + C::kStages;
    int* abort_flag = reinterpret_cast<int*>(empty + C::kStages);

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
    const int row0 = rt * 16 * W;
    if (row0 >= rows_total) return;
    const int live_warps = min(W, (rows_total - row0 + 15) / 16);
    const int j_lo = row0 / G;
    const int j_hi = min(k - 1, (row0 + 16 * W - 1) / G);
    const int min_lim = L - k + j_lo;   // smallest causal limit in the tile
    const int range_end = L - k + j_hi + 1;
    const int nchunks = (range_end + kChunk - 1) / kChunk;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], live_warps);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();

    const uint64_t pol = l2_policy_evict_first();

    if (warp == W) {
        // ------------------------------------------------------ producer
        const int32_t* bt = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
        int ids = 0;
        int issued = 0;
        for (int c = 0; c < nchunks; ++c) {
            if ((c & 31) == 0) {
                const int cc = c + lane;
                int slot = 0;
                if (cc < nchunks) {
                    const int ctok = cc * kChunk;
                    int id = bt[ctok / BS];
                    if (id < 0 || id >= p.num_blocks) {
                        report(p.error_flags, PA_DEVERR_BLOCK_ID);
                        id = 0;
                    }
                    slot = id * BS + ctok % BS;
                }
                ids = slot;
            }
            const int slot = __shfl_sync(0xffffffffu, ids, c & 31);
            const int stage = c % C::kStages;
            if (c >= C::kStages) {
                const bool ok = mbar_wait_bounded(&empty[stage], ((c / C::kStages) - 1) & 1);
                if (!__all_sync(0xffffffffu, ok) ||
                    *reinterpret_cast<volatile int*>(abort_flag)) {
                    if (lane == 0) {
                        *reinterpret_cast<volatile int*>(abort_flag) = 1;
                        report(p.error_flags, PA_DEVERR_TIMEOUT);
                    }
                    break;
                }
            }
            if (lane == 0) {
                const uint32_t dst = smem_u32(smem + stage * C::kStageBytes);
                mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h) {
                    mq_tma_load(dst + h * C::kHalfBytes, &tm_k, 0, g * C::kHalves + h,
                                slot, &full[stage], pol);
                    mq_tma_load(dst + C::kKVBytes + h * C::kHalfBytes, &tm_v, 0,
                                g * C::kHalves + h, slot, &full[stage], pol);
                }
            }
            ++issued;
        }
        // Every armed phase must land before the CTA may exit.
        for (int c = (issued > C::kStages ? issued - C::kStages : 0); c < issued; ++c)
            (void)mbar_wait_bounded(&full[c % C::kStages], (c / C::kStages) & 1);
        return;
    }
    if (warp >= live_warps) return;

    // ---------------------------------------------------------- consumer
    const int qr = lane >> 2;
    const int qc = (lane & 3) * 2;
    const int xr = lane & 7;
    const int mi = lane >> 3;
    const int R0 = row0 + warp * 16 + qr;  // this lane's two rows
    const int R1 = R0 + 8;
    const bool live0 = R0 < rows_total;
    const bool live1 = R1 < rows_total;
    const int j0 = R0 / G, j1 = R1 / G;
    const int lim0 = live0 ? L - k + j0 : -1;  // last visible token
    const int lim1 = live1 ? L - k + j1 : -1;

    uint32_t qa[D / 16][4];
    {
        const uint16_t* qp0 = p.q + ((int64_t)(q0 + (live0 ? j0 : 0)) * Hq + g * G + (live0 ? R0 % G : 0)) * D;
        const uint16_t* qp1 = p.q + ((int64_t)(q0 + (live1 ? j1 : 0)) * Hq + g * G + (live1 ? R1 % G : 0)) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = live0 ? *reinterpret_cast<const uint32_t*>(qp0 + ks * 16 + qc) : 0u;
            qa[ks][1] = live1 ? *reinterpret_cast<const uint32_t*>(qp1 + ks * 16 + qc) : 0u;
            qa[ks][2] = live0 ? *reinterpret_cast<const uint32_t*>(qp0 + ks * 16 + 8 + qc) : 0u;
            qa[ks][3] = live1 ? *reinterpret_cast<const uint32_t*>(qp1 + ks * 16 + 8 + qc) : 0u;
        }
    }

    float o[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    const float sl2 = p.scale_log2;

    for (int c = 0; c < nchunks; ++c) {
        const int stage = c % C::kStages;
        const bool ok = mbar_wait_bounded(&full[stage], (c / C::kStages) & 1);
        if (!__all_sync(0xffffffffu, ok) || *reinterpret_cast<volatile int*>(abort_flag)) {
            if (lane == 0) {
                *reinterpret_cast<volatile int*>(abort_flag) = 1;
                report(p.error_flags, PA_DEVERR_TIMEOUT);
            }
            return;
        }
        const int ctok = c * kChunk;
        const int valid = min(kChunk, range_end - ctok);
        const uint32_t kaddr = smem_u32(smem + stage * C::kStageBytes);
        const uint32_t vaddr = kaddr + C::kKVBytes;

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
                mma_bf16_16816(sacc[nt][kk & 1], qa[2 * kk][0], qa[2 * kk][1],
                               qa[2 * kk][2], qa[2 * kk][3], b0, b1);
                mma_bf16_16816(sacc[nt][kk & 1], qa[2 * kk + 1][0], qa[2 * kk + 1][1],
                               qa[2 * kk + 1][2], qa[2 * kk + 1][3], b2, b3);
            }
        }
        // sv[r][i]: row r (0: R0, 1: R1), token ctok + (i>>1)*8 + qc + (i&1)
        float sv[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                sv[r][i] = (sacc[i >> 1][0][r * 2 + (i & 1)] + sacc[i >> 1][1][r * 2 + (i & 1)]) * sl2;
        if (ctok + kChunk - 1 > min_lim) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tok = ctok + (i >> 1) * 8 + qc + (i & 1);
                if (tok > lim0) sv[0][i] = -INFINITY;
                if (tok > lim1) sv[1][i] = -INFINITY;
            }
        }
        float mx[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            mx[r] = fmaxf(fmaxf(sv[r][0], sv[r][1]), fmaxf(sv[r][2], sv[r][3]));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        }
        if (__any_sync(0xffffffffu, mx[0] > m_run[0] || mx[1] > m_run[1])) {
            float alpha[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float m_new = fmaxf(m_run[r], mx[r]);
                alpha[r] = m_new == -INFINITY ? 1.f : exp2f(m_run[r] - m_new);
                m_run[r] = m_new;
                l_run[r] *= alpha[r];
            }
#pragma unroll
            for (int j = 0; j < D / 8; ++j) {
                o[j][0] *= alpha[0]; o[j][1] *= alpha[0];
                o[j][2] *= alpha[1]; o[j][3] *= alpha[1];
            }
        }
        float pv[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                pv[r][i] = sv[r][i] == -INFINITY ? 0.f : exp2f(sv[r][i] - m_run[r]);
            l_run[r] += (pv[r][0] + pv[r][1]) + (pv[r][2] + pv[r][3]);
        }
        float hi[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) hi[r][i] = bf16_round(pv[r][i]);
        const uint32_t ah0 = pack_bf16x2(hi[0][0], hi[0][1]);
        const uint32_t ah1 = pack_bf16x2(hi[1][0], hi[1][1]);
        const uint32_t ah2 = pack_bf16x2(hi[0][2], hi[0][3]);
        const uint32_t ah3 = pack_bf16x2(hi[1][2], hi[1][3]);
        const uint32_t al0 = pack_bf16x2(pv[0][0] - hi[0][0], pv[0][1] - hi[0][1]);
        const uint32_t al1 = pack_bf16x2(pv[1][0] - hi[1][0], pv[1][1] - hi[1][1]);
        const uint32_t al2 = pack_bf16x2(pv[0][2] - hi[0][2], pv[0][3] - hi[0][3]);
        const uint32_t al3 = pack_bf16x2(pv[1][2] - hi[1][2], pv[1][3] - hi[1][3]);

        const uint32_t vrow = vaddr + (((mi & 1) << 3) + xr) * 128;
        const int tb = (lane & 3) * 2;  // token pair this lane's B halves hold
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
            const int cidx = ((dp & 3) << 1) + (mi >> 1);
            const uint32_t a = vrow + (dp >> 2) * C::kHalfBytes + ((cidx ^ xr) << 4);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_trans(b0, b1, b2, b3, a);
            if (valid < kChunk) {  // rows past the range may hold anything
                b0 = keep_tokens(b0, tb, valid);
                b1 = keep_tokens(b1, 8 + tb, valid);
                b2 = keep_tokens(b2, tb, valid);
                b3 = keep_tokens(b3, 8 + tb, valid);
            }
            mma_bf16_16816(o[2 * dp], ah0, ah1, ah2, ah3, b0, b1);
            mma_bf16_16816(o[2 * dp], al0, al1, al2, al3, b0, b1);
            mma_bf16_16816(o[2 * dp + 1], ah0, ah1, ah2, ah3, b2, b3);
            mma_bf16_16816(o[2 * dp + 1], al0, al1, al2, al3, b2, b3);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
    }

#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
        l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
    }
    if (live0) {
        float* dst = p.out + ((int64_t)(q0 + j0) * Hq + g * G + R0 % G) * D + qc;
        const float inv = 1.f / l_run[0];
#pragma unroll
        for (int j = 0; j < D / 8; ++j)
            *reinterpret_cast<float2*>(dst + 8 * j) = make_float2(o[j][0] * inv, o[j][1] * inv);
    }
    if (live1) {
        float* dst = p.out + ((int64_t)(q0 + j1) * Hq + g * G + R1 % G) * D + qc;
        const float inv = 1.f / l_run[1];
#pragma unroll
        for (int j = 0; j < D / 8; ++j)
            *reinterpret_cast<float2*>(dst + 8 * j) = make_float2(o[j][2] * inv, o[j][3] * inv);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                   void*, const cuuint64_t*, const cuuint64_t*,
                                   const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn mq_encode_fn() {
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

bool mq_encode_map(CUtensorMap* map, const void* pool, int num_blocks,
                   int block_size, int num_kv_heads, int head_size) {
    EncodeTiledFn fn = mq_encode_fn();
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

template <int D, int BS, int W>
cudaError_t mq_launch_typed(const MultiQueryParams& p, int row_tiles,
                            cudaStream_t stream) {
    using C = MQCfg<D>;
    static int ready[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE)) {
        e = cudaFuncSetAttribute(paged_multi_query_kernel<D, BS, W>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes);
        if (e != cudaSuccess) return e;
        __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
    }
    CUtensorMap tmk, tmv;
    if (!mq_encode_map(&tmk, p.k_cache, p.num_blocks, BS, p.num_kv_heads, D) ||
        !mq_encode_map(&tmv, p.v_cache, p.num_blocks, BS, p.num_kv_heads, D))
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_kv_heads, (unsigned)row_tiles,
                       (unsigned)p.num_seqs);
    cfg.blockDim = dim3((W + 1) * 32);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, paged_multi_query_kernel<D, BS, W>, tmk, tmv, p);
    count_launch();
    return e;
}

template <int D, int BS>
cudaError_t mq_launch_w(const MultiQueryParams& p, cudaStream_t stream) {
    const int rows = p.max_query_len * p.group;
    const int W = rows <= 16 ? 1 : (rows <= 32 ? 2 : 4);
    const int tiles = (rows + 16 * W - 1) / (16 * W);
    if (W == 1) return mq_launch_typed<D, BS, 1>(p, tiles, stream);
    if (W == 2) return mq_launch_typed<D, BS, 2>(p, tiles, stream);
    return mq_launch_typed<D, BS, 4>(p, tiles, stream);
}

}  // namespace

int multi_query_row_tiles(int max_query_len, int group) {
    const int rows = max_query_len * group;
    const int W = rows <= 16 ? 1 : (rows <= 32 ? 2 : 4);
    return (rows + 16 * W - 1) / (16 * W);
}

cudaError_t launch_paged_multi_query(const MultiQueryParams& p, int head_size,
                                     int block_size, cudaStream_t stream) {
    if (head_size == 128 && block_size == 16) return mq_launch_w<128, 16>(p, stream);
    if (head_size == 128 && block_size == 32) return mq_launch_w<128, 32>(p, stream);
    if (head_size == 64 && block_size == 16) return mq_launch_w<64, 16>(p, stream);
    if (head_size == 64 && block_size == 32) return mq_launch_w<64, 32>(p, stream);
    return cudaErrorInvalidValue;
}

float mq_log2e_scale(float scale) { return scale * kLog2e; }

}  // namespace pa
