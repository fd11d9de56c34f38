// Block statistics on tcgen05 tensor cores (bf16 inputs).
//
// Per key block j (PISA paper, section 3.4 and Figure 3, the prepare phase;
// "Sparse Linear Attention" blog, sections "Sparse Linear Attention" and "Going
// Further: Adding the Second-Order Term (PWT)"):
//   kbar_j = (1/B) sum_n k_n          canonical fp32 pairwise tree (CUDA cores)
//   vsum_j = sum_n v_n                fp32 (CUDA cores)
//   H_j    = sum_n v_n (k_n - kbar_j)^T = V_j^T K_j - vsum_j kbar_j^T
//   C_j    = (1/B) sum_n (k_n - kbar_j)(k_n - kbar_j)^T = (1/B) K_j^T K_j - kbar_j kbar_j^T
// The two Gram products run on the tensor cores straight from the token tiles:
// V_j^T and K_j^T are read as MN-major A operands, K_j as the MN-major B
// operand (both K-dimensions are the B tokens), fp32 accumulation in TMEM; the
// rank-1 corrections and the 1/B are applied in fp32 in the epilogue.  For
// d = 64 the A operand is [V_j^T ; K_j^T] stacked to M = 128, so one MMA gives
// H_j (rows 0-63) and the uncentred C_j (rows 64-127).
//
// With kaug non-null it also writes, per block, the eight bf16 rows the
// statistics-form tensor-core kernel appends to H_j as extra B-operand rows:
// row 0 = bf16(kbar_j) (round to nearest), row 1 = bf16(kbar_j - row 0), rows
// 2-7 = 0, so that one MMA gives q . kbar_j as two columns to within about
// 2^-16 of the fp32 centroid.
//
// One CTA (128 threads) per (block, bh): warp 0 allocates TMEM, lane 0 of
// warp 0 issues the TMA loads and the MMAs; all four warps then compute the
// column sums from shared memory and run the epilogue (thread = TMEM lane).
#pragma once

#include <cudaTypedefs.h>

#include <string>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace pisa {

template <int D, int BS>
struct StatsTcCfg {
    static constexpr uint32_t BOX_BYTES = BS * 128;             // BS rows x 64 bf16 columns
    static constexpr uint32_t TILE_BYTES = (D / 64) * BOX_BYTES;
    static constexpr uint32_t V_OFF = 0;                        // V tile first: [V ; K] stacking for d = 64
    static constexpr uint32_t K_OFF = TILE_BYTES;
    static constexpr uint32_t BAR_OFF = 2 * TILE_BYTES;
    static constexpr uint32_t KB_OFF = BAR_OFF + 64;            // fp32 kbar[D], vsum[D]
    static constexpr uint32_t SMEM = KB_OFF + 2 * D * 4 + 1024;
};

template <int D, int ORDER>
constexpr uint32_t stats_tmem_cols() { return D == 128 ? (ORDER == 2 ? 256u : 128u) : 64u; }

// bf16 element (n, c) of a tile staged by TMA with 128-byte swizzle in boxes of
// 64 columns: 16-byte chunk index XOR (row mod 8).
template <int BS>
__device__ __forceinline__ float swz_elem(const uint8_t* tile, int n, int c) {
    const int box = c >> 6, cc = c & 63;
    const int chunk = (cc >> 3) ^ (n & 7);
    const bf16* p = reinterpret_cast<const bf16*>(tile + box * (BS * 128) + n * 128 + chunk * 16) + (cc & 7);
    return __bfloat162float(*p);
}

template <int D, int BS, int ORDER>
__global__ void __launch_bounds__(128) stats_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                       const __grid_constant__ CUtensorMap tm_v,
                                                       float* __restrict__ kbar, float* __restrict__ vsum,
                                                       bf16* __restrict__ hstat, bf16* __restrict__ cov,
                                                       bf16* __restrict__ kaug, int L, int nblk, unsigned* status) {
    using C = StatsTcCfg<D, BS>;
    // M = 128 always (d = 64 stacks V and K); N = d; both operands MN-major
    constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                               ((uint32_t)(D >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_addr(smem);
    const uint32_t bar_full = sbase + C::BAR_OFF, bar_mma = sbase + C::BAR_OFF + 8;
    uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + 16);
    float* kb = (float*)(smem + C::KB_OFF);
    float* vs = kb + D;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int j = blockIdx.x, bh = blockIdx.y;
    bool aborted = false;

    if (threadIdx.x == 0) {
        tc::mbar_init(bar_full, 1);
        tc::mbar_init(bar_mma, 1);
        tc::fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), stats_tmem_cols<D, ORDER>());
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (threadIdx.x == 0) {
        const int row = bh * L + j * BS;
        tc::mbar_expect_tx(bar_full, 2 * C::TILE_BYTES);
        for (int b = 0; b < D / 64; ++b) {
            tc::tma_load_2d(sbase + C::V_OFF + b * C::BOX_BYTES, &tm_v, bar_full, b * 64, row);
            tc::tma_load_2d(sbase + C::K_OFF + b * C::BOX_BYTES, &tm_k, bar_full, b * 64, row);
        }
        if (tc::mbar_wait(bar_full, 0, aborted, status, 2000000000ll)) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < BS / 16; ++kk) {
                const uint32_t off = kk * 16 * 128;  // 16 tokens further along K
                // H_raw (d = 128), or [H_raw ; C_raw] (d = 64): A = V^T (stacked with K^T)
                const uint64_t a_v = tc::sdesc_sw128(sbase + C::V_OFF + off, C::BOX_BYTES, 1024);
                const uint64_t b_k = tc::sdesc_sw128(sbase + C::K_OFF + off, C::BOX_BYTES, 1024);
                tc::mma_ss(tmem, a_v, b_k, IDESC, kk > 0);
                if (D == 128 && ORDER == 2) {
                    const uint64_t a_k = tc::sdesc_sw128(sbase + C::K_OFF + off, C::BOX_BYTES, 1024);
                    tc::mma_ss(tmem + 128, a_k, b_k, IDESC, kk > 0);
                }
            }
            tc::mma_commit(bar_mma);
        }
    }
    // column sums from shared memory (all threads), once the tiles have landed
    if (tc::mbar_wait_warp(bar_full, 0, aborted, status, 2000000000ll)) {
        for (int c = threadIdx.x; c < D; c += 128) {
            float a[BS];
#pragma unroll
            for (int n = 0; n < BS; ++n) a[n] = swz_elem<BS>(smem + C::K_OFF, n, c);
            const float m = __fmul_rn(tree_sum<BS>(a), 1.0f / (float)BS);
            float s = 0.f;
            for (int n = 0; n < BS; ++n) s += swz_elem<BS>(smem + C::V_OFF, n, c);
            kb[c] = m;
            vs[c] = s;
            const size_t so = ((size_t)bh * nblk + j) * D + c;
            kbar[so] = m;
            vsum[so] = s;
            if (kaug) {
                bf16* ka = kaug + ((size_t)bh * nblk + j) * 8 * D + c;
                const bf16 hi = __float2bfloat16_rn(m);
                ka[0] = hi;
                ka[D] = __float2bfloat16_rn(m - __bfloat162float(hi));
#pragma unroll
                for (int rr = 2; rr < 8; ++rr) ka[rr * D] = __float2bfloat16_rn(0.f);
            }
        }
    }
    __syncthreads();
    if (tc::mbar_wait_warp(bar_mma, 0, aborted, status, 2000000000ll)) {
        tc::fence_after_sync();
        const int r = warp * 32 + lane;  // TMEM lane = output row
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
        const size_t base = ((size_t)bh * nblk + j) * D * D;
        const float inv_b = 1.0f / (float)BS;
        // which matrix and row this lane holds
        const bool is_h = (D == 128) || (r < 64);
        const int a = (D == 128) ? r : (r & 63);
        const bool want = is_h || ORDER == 2;
        const float rowv = is_h ? vs[a] : kb[a];
#pragma unroll
        for (int part = 0; part < ((D == 128 && ORDER == 2) ? 2 : 1); ++part) {
            const bool h_here = (D == 128) ? (part == 0) : is_h;
            bf16* dst = (h_here ? hstat : cov) + base + (size_t)a * D;
            const float rv = (D == 128) ? (part == 0 ? vs[a] : kb[a]) : rowv;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t raw[32];
                tc::tmem_ld32(taddr + part * 128 + c0, raw);
                tc::tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float x0 = __uint_as_float(raw[2 * e]), x1 = __uint_as_float(raw[2 * e + 1]);
                    if (h_here) {
                        x0 = fmaf(-rv, kb[c0 + 2 * e], x0);
                        x1 = fmaf(-rv, kb[c0 + 2 * e + 1], x1);
                    } else {
                        x0 = fmaf(-rv, kb[c0 + 2 * e], x0 * inv_b);
                        x1 = fmaf(-rv, kb[c0 + 2 * e + 1], x1 * inv_b);
                    }
                    pk[e] = tc::pack_bf16x2(x0, x1);
                }
                if (want) {
                    uint4* o = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, stats_tmem_cols<D, ORDER>());
    }
}

inline pisa_status run_stats_tc(const void* k, const void* v, float* kbar, float* vsum, void* hstat, void* cov,
                                void* kaug, long BH, int L, int d, int B, int nblk, int order, unsigned* status,
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
        CUresult cr = encode(&maps[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptrs[t]), gdim, gstride,
                             box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS) {
            *err = "cuTensorMapEncodeTiled failed (" + std::to_string((int)cr) + ")";
            return PISA_ERR_CUDA;
        }
    }
    dim3 grid((unsigned)nblk, (unsigned)BH);
    cudaError_t e = cudaSuccess;
#define PISA_STATS_TC(DD, BB, OO)                                                                             \
    if (d == DD && B == BB && order == OO) {                                                                  \
        auto kern = stats_tc_kernel<DD, BB, OO>;                                                              \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,                           \
                                 (int)StatsTcCfg<DD, BB>::SMEM);                                              \
        if (e == cudaSuccess) {                                                                               \
            kern<<<grid, 128, StatsTcCfg<DD, BB>::SMEM, s>>>(maps[0], maps[1], kbar, vsum, (bf16*)hstat,      \
                                                             (bf16*)cov, (bf16*)kaug, L, nblk, status);       \
            e = cudaGetLastError();                                                                           \
        }                                                                                                     \
    } else
    PISA_STATS_TC(64, 64, 1)
    PISA_STATS_TC(64, 64, 2)
    PISA_STATS_TC(64, 128, 1)
    PISA_STATS_TC(64, 128, 2)
    PISA_STATS_TC(128, 64, 1)
    PISA_STATS_TC(128, 64, 2)
    PISA_STATS_TC(128, 128, 1)
    PISA_STATS_TC(128, 128, 2) {
        *err = "no tensor-core statistics kernel for this d/B/order";
        return PISA_ERR_UNSUPPORTED;
    }
#undef PISA_STATS_TC
    if (e != cudaSuccess) {
        *err = std::string("stats_tc_kernel launch: ") + cudaGetErrorString(e);
        return PISA_ERR_CUDA;
    }
    return PISA_OK;
}

}  // namespace pisa
