// Prepare phase of the PISA hybrid (global first-order statistic).
//
// PISA paper, Figure 3 caption and section 3.4 ("block-wise means of queries and
// keys, block-wise sums of values and the global statistic H-bar in a single
// pass"); H-bar as defined in the "Sparse Linear Attention" blog, section
// "Sparse Linear Attention": H-bar = (B/L) sum_j H_j with
// H_j = sum_n v_n (k_n - kbar_j)^T = V_j^T K_j - vsum_j kbar_j^T.
//
// One CTA (128 threads) per (chunk of G consecutive blocks, bh), K_j and V_j
// staged by TMA through two stages.  Per block:
//   - canonical fp32 centroid (the selection's) and value sum, from shared
//     memory; written as fp32 (centroid) and bf16 (centroid and value sum, the
//     virtual-token operands of the hybrid attention kernel);
//   - V_j^T K_j accumulated over the chunk in TMEM (tcgen05, MN-major operands
//     straight from the token tiles; d = 64 stacks [V ; K] to M = 128);
//   - vsum_j kbar_j^T accumulated over the chunk in fp32 registers (thread a
//     holds row a).
// At the end each thread writes (B/L) (TMEM row - register row), the chunk's
// share of H-bar, to the chunk's own fp32 slot; hbar_reduce_kernel then sums
// the slots of each (batch, head) in chunk order and rounds to bf16, so H-bar
// (and the hybrid's output) is the same on every run.
#pragma once

#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "stats_tc.cuh"  // swz_elem

#include <string>

namespace pisa {

template <int D, int BS>
struct HybPrepCfg {
    static constexpr uint32_t BOX_BYTES = BS * 128;
    static constexpr uint32_t TILE_BYTES = (D / 64) * BOX_BYTES;
    static constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;  // V tile, then K tile
    static constexpr uint32_t BAR_OFF = 2 * STAGE_BYTES;
    static constexpr uint32_t KB_OFF = BAR_OFF + 64;
    static constexpr uint32_t SMEM = KB_OFF + 2 * D * 4 + 1024;
    static constexpr uint32_t TMEM_COLS = (D == 128) ? 128 : 64;
};

template <int D, int BS>
__global__ void __launch_bounds__(128, 1) hybrid_prep_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, float* __restrict__ kbar,
    bf16* __restrict__ kbar_bf, bf16* __restrict__ vsum_bf, float* __restrict__ hbar_part, int L, int nblk, int G,
    float scale, unsigned* status) {
    using C = HybPrepCfg<D, BS>;
    constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                               ((uint32_t)(D >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    constexpr long long LIMIT = 2000000000ll;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_addr(smem);
    const uint32_t bar_full0 = sbase + C::BAR_OFF, bar_mma = sbase + C::BAR_OFF + 16;
    uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + 24);
    float* kb = (float*)(smem + C::KB_OFF);
    float* vs = kb + D;
    const int tid = threadIdx.x, warp = tid / 32;
    const int bh = blockIdx.y;
    const int j0 = blockIdx.x * G;
    const int ng = min(G, nblk - j0);
    bool aborted = false;

    if (tid == 0) {
        tc::mbar_init(bar_full0, 1);
        tc::mbar_init(bar_full0 + 8, 1);
        tc::mbar_init(bar_mma, 1);
        tc::fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    auto load_block = [&](int i) {
        const int s = i & 1;
        const int row = bh * L + (j0 + i) * BS;
        const uint32_t st = sbase + s * C::STAGE_BYTES;
        tc::mbar_expect_tx(bar_full0 + 8 * s, C::STAGE_BYTES);
        for (int b = 0; b < D / 64; ++b) {
            tc::tma_load_2d(st + b * C::BOX_BYTES, &tm_v, bar_full0 + 8 * s, b * 64, row);
            tc::tma_load_2d(st + C::TILE_BYTES + b * C::BOX_BYTES, &tm_k, bar_full0 + 8 * s, b * 64, row);
        }
    };
    if (tid == 0) {
        tc::tma_prefetch(&tm_k);
        tc::tma_prefetch(&tm_v);
        load_block(0);
        if (ng > 1) load_block(1);
    }

    float R[D];  // row `tid` of sum_j vsum_j kbar_j^T (rows < D hold H rows)
#pragma unroll
    for (int b = 0; b < D; ++b) R[b] = 0.f;

    for (int i = 0; i < ng; ++i) {
        const int s = i & 1;
        const uint8_t* st = smem + s * C::STAGE_BYTES;
        if (!tc::mbar_wait_warp(bar_full0 + 8 * s, (i >> 1) & 1, aborted, status, LIMIT)) break;
        const int j = j0 + i;
        for (int c = tid; c < D; c += 128) {
            float a[BS];
#pragma unroll
            for (int n = 0; n < BS; ++n) a[n] = swz_elem<BS>(st + C::TILE_BYTES, n, c);
            const float m = __fmul_rn(tree_sum<BS>(a), 1.0f / (float)BS);
            float sv = 0.f;
            for (int n = 0; n < BS; ++n) sv += swz_elem<BS>(st, n, c);
            kb[c] = m;
            vs[c] = sv;
            const size_t o = ((size_t)bh * nblk + j) * D + c;
            kbar[o] = m;
            kbar_bf[o] = __float2bfloat16_rn(m);
            vsum_bf[o] = __float2bfloat16_rn(sv);
        }
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t sa = sbase + s * C::STAGE_BYTES;
#pragma unroll
            for (int kk = 0; kk < BS / 16; ++kk) {
                const uint32_t off = kk * 16 * 128;
                tc::mma_ss(tmem, tc::sdesc_sw128(sa + off, C::BOX_BYTES, 1024),
                           tc::sdesc_sw128(sa + C::TILE_BYTES + off, C::BOX_BYTES, 1024), IDESC,
                           (i > 0 || kk > 0) ? 1u : 0u);
            }
            tc::mma_commit(bar_mma);
            // the stage may be refilled only once the tensor core has read it
            if (tc::mbar_wait(bar_mma, i & 1, aborted, status, LIMIT) && i + 2 < ng) load_block(i + 2);
        }
        if (tid < D) {
            const float va = vs[tid];
#pragma unroll
            for (int b = 0; b < D; ++b) R[b] = fmaf(va, kb[b], R[b]);
        }
        __syncthreads();
    }

    // every MMA has completed (thread 0 waited for each); this chunk's (B/L)(V^T K - R)
    tc::fence_after_sync();
    if (!aborted) {
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
        float* dst = hbar_part + (((size_t)bh * gridDim.x + blockIdx.x) * D + (tid < D ? tid : 0)) * D;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t raw[32];
            tc::tmem_ld32(taddr + c0, raw);
            tc::tmem_wait_ld();
            if (tid < D) {
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4*>(dst + c0 + e) =
                        make_float4(scale * (__uint_as_float(raw[e]) - R[c0 + e]),
                                    scale * (__uint_as_float(raw[e + 1]) - R[c0 + e + 1]),
                                    scale * (__uint_as_float(raw[e + 2]) - R[c0 + e + 2]),
                                    scale * (__uint_as_float(raw[e + 3]) - R[c0 + e + 3]));
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// H-bar = sum of the chunks' slots in chunk order (fixed, so reproducible), rounded to bf16
// (row = value channel, the K-major B operand of Q H-bar^T).  part: [BH, nchunk, d*d].
__global__ void hbar_reduce_kernel(const float* __restrict__ part, bf16* __restrict__ out, long BH, int nchunk,
                                   int dd) {
    const long n = BH * (long)dd;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const long bh = i / dd, e = i % dd;
        const float* p = part + (size_t)bh * nchunk * dd + e;
        float acc = 0.f;
        for (int c = 0; c < nchunk; ++c) acc += p[(size_t)c * dd];
        out[i] = __float2bfloat16_rn(acc);
    }
}

// Blocks per CTA of the prepare kernel: 64, halved (down to 8) until the grid has
// about four CTAs per SM.  The number of chunks (CTAs per head) sizes H-bar's slots.
inline int hybrid_prep_chunk(long BH, int nblk) {
    int G = 64;
    while (G > 8 && (long)((nblk + G - 1) / G) * BH < 4L * 148) G /= 2;
    return G;
}
inline int hybrid_prep_nchunk(long BH, int nblk) {
    const int G = hybrid_prep_chunk(BH, nblk);
    return (nblk + G - 1) / G;
}

// Host: tensor maps, the prepare kernel and the ordered reduction of H-bar.
// hpart: [BH, hybrid_prep_nchunk(BH, nblk), d, d] fp32 (every slot is written).
inline pisa_status run_hybrid_prep(const void* k, const void* v, float* kbar, bf16* kbar_bf, bf16* vsum_bf,
                                   float* hpart, bf16* hbf, long BH, int L, int d, int B, int nblk, unsigned* status,
                                   cudaStream_t s, std::string* err) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess || !fn) {
            *err = "cuTensorMapEncodeTiled not available";
            return PISA_ERR_CUDA;
        }
        encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    }
    CUtensorMap maps[2];
    const void* ptrs[2] = {k, v};
    for (int t = 0; t < 2; ++t) {
        cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)(BH * L)};
        cuuint64_t gstride[1] = {(cuuint64_t)d * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)B};
        cuuint32_t estride[2] = {1, 1};
        if (encode(&maps[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptrs[t]), gdim, gstride, box,
                   estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
            *err = "cuTensorMapEncodeTiled failed for the hybrid prepare kernel";
            return PISA_ERR_CUDA;
        }
    }
    const int G = hybrid_prep_chunk(BH, nblk);
    const int nchunk = (nblk + G - 1) / G;
    dim3 grid((unsigned)nchunk, (unsigned)BH);
    const float scale = (float)B / (float)L;
    cudaError_t e = cudaSuccess;
#define PISA_HPREP(DD, BB)                                                                                     \
    if (d == DD && B == BB) {                                                                                  \
        auto kern = hybrid_prep_kernel<DD, BB>;                                                                \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)HybPrepCfg<DD, BB>::SMEM); \
        if (e == cudaSuccess) {                                                                                \
            kern<<<grid, 128, HybPrepCfg<DD, BB>::SMEM, s>>>(maps[0], maps[1], kbar, kbar_bf, vsum_bf, hpart, L, nblk, \
                                                             G, scale, status);                                \
            e = cudaGetLastError();                                                                            \
        }                                                                                                      \
    } else
    PISA_HPREP(64, 64)
    PISA_HPREP(64, 128)
    PISA_HPREP(128, 64)
    PISA_HPREP(128, 128) {
        *err = "no hybrid prepare kernel for this d/B";
        return PISA_ERR_UNSUPPORTED;
    }
#undef PISA_HPREP
    if (e != cudaSuccess) {
        *err = std::string("hybrid_prep_kernel launch: ") + cudaGetErrorString(e);
        return PISA_ERR_CUDA;
    }
    const long n = BH * (long)d * d;
    hbar_reduce_kernel<<<(unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0, s>>>(hpart, hbf, BH,
                                                                                                 nchunk, d * d);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        *err = std::string("hbar_reduce_kernel launch: ") + cudaGetErrorString(e);
        return PISA_ERR_CUDA;
    }
    return PISA_OK;
}

}  // namespace pisa
