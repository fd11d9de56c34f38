// Covariance-aware routing bias: bias_j = ln(||H_j||_F + eps) per key block.
//
// PISA paper, section 3.3 "Covariance-Aware Block Selection" (the log of a
// block norm plus eps is added to the centroid score before the top-K);
// "Sparse Linear Attention" blog, PWT section (route by the block score plus
// the log of the norm of H_j).  The bias decides which blocks are selected, so
// it follows a canonical fp32 procedure that any implementation reproduces bit
// for bit:
//   kbar_j[c]  = the selection's canonical centroid (input)
//   dev[n][b]  = k_{j,n}[b] - kbar_j[b]
//   h[a*d + b] = tree sum over n of (v_{j,n}[a] * dev[n][b])   (H_j, value channel a)
//   M_j        = sqrt(tree sum over a*d + b of h^2)
//   bias_j     = ln_repro(M_j + eps)
// where a tree sum over a power-of-two count pairs element i with i + h for
// h = n/2, n/4, ..., 1, every product and sum is one IEEE round-to-nearest
// fp32 operation, and ln_repro is the fixed-operation logarithm below.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace pisa {

// Natural logarithm from a fixed sequence of IEEE fp32 operations (so that
// every implementation gets the same bits): x = 2^e m with m folded into
// [sqrt(1/2), sqrt(2)); ln m = 2 atanh(s), s = (m - 1)/(m + 1), by the odd
// series s + s^3/3 + s^5/5 + s^7/7 + s^9/9 (|s| <= 0.1716: truncation below
// 2e-10 relative), evaluated by Horner in s^2; ln x = e ln 2 + ln m.  For
// finite x > 0 in the normal range.
__device__ __forceinline__ float ln_repro(float x) {
    const uint32_t bits = __float_as_uint(x);
    int e = (int)((bits >> 23) & 0xffu) - 127;
    float m = __uint_as_float((bits & 0x007fffffu) | 0x3f800000u);  // [1, 2)
    if (m > 0x1.6a09e6p+0f) {  // fp32 sqrt(2); halving is exact
        m = __fmul_rn(m, 0.5f);
        e += 1;
    }
    const float s = __fdiv_rn(__fsub_rn(m, 1.0f), __fadd_rn(m, 1.0f));
    const float s2 = __fmul_rn(s, s);
    float t = __fmul_rn(0x1.c71c72p-4f, s2);  // fp32 1/9, 1/7, 1/5, 1/3
    t = __fadd_rn(t, 0x1.24924ap-3f);
    t = __fmul_rn(t, s2);
    t = __fadd_rn(t, 0x1.99999ap-3f);
    t = __fmul_rn(t, s2);
    t = __fadd_rn(t, 0x1.555556p-2f);
    t = __fmul_rn(t, s2);
    t = __fadd_rn(t, 1.0f);
    const float lnm = __fmul_rn(__fmul_rn(t, s), 2.0f);
    return __fadd_rn(__fmul_rn(__int2float_rn(e), 0x1.62e43p-1f), lnm);  // fp32 ln 2
}

template <int D, int BS>
struct RouteCfg {
    static constexpr int THREADS = 256;
    static constexpr int NE = D * D / THREADS;  // H entries per thread (e = tid + 256 m, one key channel)
    static constexpr int VS = BS + 4;            // row stride of the transposed values (16-byte rows)
    static constexpr size_t SMEM = sizeof(float) * ((size_t)D * VS + (size_t)D * D);
};

// One CTA per (key block j, bh).  Thread tid computes the entries
// e = tid + 256 m of H_j, which all share the key channel b = e mod d: its B
// deviations dev[n][b] stay in registers, and the values are read transposed
// (vT[a][n]) with 16-byte loads that the whole warp shares (a is the same for
// all lanes of a warp).  Scalar IEEE operations only (__fmul_rn / __fadd_rn,
// never fused; packed fp32x2 arithmetic does not reproduce separately rounded
// scalar operations).  The squares go to shared memory and the canonical tree
// over all d^2 of them runs there.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(256) route_bias_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                                         const float* __restrict__ kbar, int L, int nblk,
                                                         float eps, float* __restrict__ bias) {
    using C = RouteCfg<D, BS>;
    extern __shared__ __align__(16) float sm_route[];
    float* vT = sm_route;          // [D][VS]: vT[a][n] = v_{j,n}[a]
    float* sq = vT + D * C::VS;    // [D * D]
    const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const size_t base = ((size_t)bh * L + (size_t)j * BS) * D;
    for (int e = tid; e < BS * D; e += C::THREADS) vT[(e % D) * C::VS + e / D] = to_f(v[base + e]);
    const int b = tid % D;
    float dv[BS];  // dev[n][b] = k_{j,n}[b] - kbar_j[b]
    {
        const float kb = kbar[((size_t)bh * nblk + j) * D + b];
#pragma unroll
        for (int n = 0; n < BS; ++n) dv[n] = __fsub_rn(to_f(k[base + (size_t)n * D + b]), kb);
    }
    __syncthreads();
#pragma unroll 1
    for (int m = 0; m < C::NE; ++m) {
        const int e = tid + C::THREADS * m;
        const float4* va = reinterpret_cast<const float4*>(vT + (e / D) * C::VS);
        // first tree level pairs n with n + BS/2
        float p[BS / 2];
#pragma unroll
        for (int i = 0; i < BS / 8; ++i) {
            const float4 lo = va[i], hi = va[BS / 8 + i];
            p[4 * i + 0] = __fadd_rn(__fmul_rn(lo.x, dv[4 * i + 0]), __fmul_rn(hi.x, dv[BS / 2 + 4 * i + 0]));
            p[4 * i + 1] = __fadd_rn(__fmul_rn(lo.y, dv[4 * i + 1]), __fmul_rn(hi.y, dv[BS / 2 + 4 * i + 1]));
            p[4 * i + 2] = __fadd_rn(__fmul_rn(lo.z, dv[4 * i + 2]), __fmul_rn(hi.z, dv[BS / 2 + 4 * i + 2]));
            p[4 * i + 3] = __fadd_rn(__fmul_rn(lo.w, dv[4 * i + 3]), __fmul_rn(hi.w, dv[BS / 2 + 4 * i + 3]));
        }
        const float h = tree_sum<BS / 2>(p);
        sq[e] = __fmul_rn(h, h);
    }
    __syncthreads();
#pragma unroll 1
    for (int h = D * D / 2; h >= 1; h /= 2) {
        for (int i = tid; i < h; i += C::THREADS) sq[i] = __fadd_rn(sq[i], sq[i + h]);
        __syncthreads();
    }
    if (tid == 0) bias[(size_t)bh * nblk + j] = ln_repro(__fadd_rn(__fsqrt_rn(sq[0]), eps));
}

}  // namespace pisa
