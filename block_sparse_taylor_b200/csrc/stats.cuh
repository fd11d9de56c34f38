// Prepare phase: per key block j of B tokens, the centroid kbar_j, the value
// sum vsum_j, the first-order cross statistic H_j and the key covariance C_j.
//
// PISA paper, section 3.4 and Figure 3 (centroids and value sums computed in
// one pass before the fused kernel); "Sparse Linear Attention" blog, section
// "Sparse Linear Attention" (H_j = sum_n v_n (k_n - kbar_j)^T) and section
// "Going Further: Adding the Second-Order Term (PWT)" (C_j, the within-block
// key covariance with the 1/B normalisation).
#pragma once

#include "common.cuh"

namespace pisa {

// Centroid of every key block in the canonical fp32 order.  One CTA per
// (block, bh): the B x D tile is staged in shared memory with 16-byte loads,
// then the thread of column c reduces its B values with the pairwise tree; the
// mean is the tree sum times 1/B (exact for B = 2^k).  grid (nblk, BH), 128
// threads, BS * D * sizeof(T) bytes of dynamic shared memory.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(128) centroid_kernel(const T* __restrict__ k, float* __restrict__ kbar,
                                                       int L, int nblk) {
    extern __shared__ __align__(16) uint8_t sm_cent[];
    T* tile = reinterpret_cast<T*>(sm_cent);
    const int j = blockIdx.x, bh = blockIdx.y;
    const uint4* src = reinterpret_cast<const uint4*>(k + ((size_t)bh * L + (size_t)j * BS) * D);
    uint4* dst = reinterpret_cast<uint4*>(tile);
    constexpr int NV = BS * D * (int)sizeof(T) / 16;
#pragma unroll 4
    for (int e = threadIdx.x; e < NV; e += 128) dst[e] = __ldg(src + e);
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += 128) {
        float a[BS];
#pragma unroll
        for (int n = 0; n < BS; ++n) a[n] = to_f(tile[n * D + c]);
        kbar[((size_t)bh * nblk + j) * D + c] = __fmul_rn(tree_sum<BS>(a), 1.0f / (float)BS);
    }
}

// Full statistics on CUDA cores.  One CTA per (block, bh), 256 threads.
// The keys are centred in shared memory with the canonical centroid, then
// H_j[a][b] = sum_n v[n][a] dev[n][b] and C_j[a][b] = (1/B) sum_n dev[n][a] dev[n][b]
// are accumulated in fp32; each thread owns a (D/16) x (D/16) tile of outputs
// with rows a = a0 + 16*i and columns b = b0 + 16*i' (conflict-free reads).
template <typename T, int D, int BS>
__global__ void __launch_bounds__(256) stats_simt_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                                         float* __restrict__ kbar, float* __restrict__ vsum,
                                                         T* __restrict__ hstat, T* __restrict__ cov, int L,
                                                         int nblk, int order) {
    constexpr int S = D + 1;  // padded fp32 row stride
    constexpr int R = D / 16;
    extern __shared__ __align__(16) float sm_stats[];
    float* ks = sm_stats;       // [BS][S] keys, then deviations
    float* vs = ks + BS * S;    // [BS][S]
    float* kb = vs + BS * S;    // [D]
    const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const size_t base = ((size_t)bh * L + (size_t)j * BS) * D;
    for (int e = tid; e < BS * D; e += 256) {
        const int n = e / D, c = e % D;
        ks[n * S + c] = to_f(k[base + e]);
        vs[n * S + c] = to_f(v[base + e]);
    }
    __syncthreads();
    const size_t so = ((size_t)bh * nblk + j) * D;
    if (tid < D) {
        float a[BS];
#pragma unroll
        for (int n = 0; n < BS; ++n) a[n] = ks[n * S + tid];
        const float m = __fmul_rn(tree_sum<BS>(a), 1.0f / (float)BS);
        kb[tid] = m;
        kbar[so + tid] = m;
        float s = 0.f;
        for (int n = 0; n < BS; ++n) s += vs[n * S + tid];
        vsum[so + tid] = s;
    }
    __syncthreads();
    if (order == 0) return;
    for (int e = tid; e < BS * D; e += 256) {
        const int n = e / D, c = e % D;
        ks[n * S + c] -= kb[c];
    }
    __syncthreads();
    const int a0 = tid / 16, b0 = tid % 16;
    float h[R][R], cv[R][R];
#pragma unroll
    for (int x = 0; x < R; ++x)
#pragma unroll
        for (int y = 0; y < R; ++y) h[x][y] = cv[x][y] = 0.f;
    const bool want_c = (order == 2);
    for (int n = 0; n < BS; ++n) {
        float va[R], da[R], db[R];
#pragma unroll
        for (int x = 0; x < R; ++x) {
            va[x] = vs[n * S + a0 + 16 * x];
            da[x] = ks[n * S + a0 + 16 * x];
            db[x] = ks[n * S + b0 + 16 * x];
        }
#pragma unroll
        for (int x = 0; x < R; ++x)
#pragma unroll
            for (int y = 0; y < R; ++y) h[x][y] = fmaf(va[x], db[y], h[x][y]);
        if (want_c) {
#pragma unroll
            for (int x = 0; x < R; ++x)
#pragma unroll
                for (int y = 0; y < R; ++y) cv[x][y] = fmaf(da[x], db[y], cv[x][y]);
        }
    }
    const size_t ho = ((size_t)bh * nblk + j) * D * D;
#pragma unroll
    for (int x = 0; x < R; ++x)
#pragma unroll
        for (int y = 0; y < R; ++y) {
            const int a = a0 + 16 * x, b = b0 + 16 * y;
            hstat[ho + a * D + b] = from_f<T>(h[x][y]);
            if (want_c) cov[ho + a * D + b] = from_f<T>(cv[x][y] * (1.0f / (float)BS));
        }
}

}  // namespace pisa

namespace pisa {

// Column statistics of every B-row tile for PWT's cheap second-order term
// ("Sparse Linear Attention" blog, PWT section): MODE 1 = within-block variance
// of each channel of the keys, (1/B) sum_n (k_nc - mean_c)^2 (the diagonal of
// C_j, two passes in fp32); MODE 2 = mean of the squared queries of a tile,
// (1/B) sum_t q_tc^2 (square first, then average).  Same staging as the
// centroid kernel; grid (nblk, BH), 128 threads.
template <typename T, int D, int BS, int MODE>
__global__ void __launch_bounds__(128) colstat_kernel(const T* __restrict__ x, float* __restrict__ out, int L,
                                                      int nblk) {
    extern __shared__ __align__(16) uint8_t sm_col[];
    T* tile = reinterpret_cast<T*>(sm_col);
    const int j = blockIdx.x, bh = blockIdx.y;
    const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)bh * L + (size_t)j * BS) * D);
    uint4* dst = reinterpret_cast<uint4*>(tile);
    constexpr int NV = BS * D * (int)sizeof(T) / 16;
#pragma unroll 4
    for (int e = threadIdx.x; e < NV; e += 128) dst[e] = __ldg(src + e);
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += 128) {
        float r;
        if (MODE == 1) {
            float m = 0.f;
            for (int n = 0; n < BS; ++n) m += to_f(tile[n * D + c]);
            m *= 1.0f / (float)BS;
            float v = 0.f;
            for (int n = 0; n < BS; ++n) {
                const float dv = to_f(tile[n * D + c]) - m;
                v = fmaf(dv, dv, v);
            }
            r = v * (1.0f / (float)BS);
        } else {
            float s = 0.f;
            for (int n = 0; n < BS; ++n) {
                const float xv = to_f(tile[n * D + c]);
                s = fmaf(xv, xv, s);
            }
            r = s * (1.0f / (float)BS);
        }
        out[((size_t)bh * nblk + j) * D + c] = r;
    }
}

// The [query tile x key block] matrix of PWT's cheap second-order term:
// w_ij = 1/2 sum_c q2_ic var_jc, set to 0 when it exceeds ln B and the gate is
// on.  grid (nblk, BH) over query tiles i, 256 threads: one warp per block j,
// lanes over channels.
template <int D>
__global__ void __launch_bounds__(256) wpool_kernel(const float* __restrict__ q2, const float* __restrict__ var,
                                                    float* __restrict__ w, int nblk, int gate, float ln_b) {
    __shared__ float qs[D];
    const int i = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    for (int c = threadIdx.x; c < D; c += 256) qs[c] = q2[((size_t)bh * nblk + i) * D + c];
    __syncthreads();
    const float* vb = var + (size_t)bh * nblk * D;
    float* wrow = w + ((size_t)bh * nblk + i) * nblk;
    for (int j = warp; j < nblk; j += 8) {
        float s = 0.f;
#pragma unroll
        for (int c = lane; c < D; c += 32) s = fmaf(qs[c], vb[(size_t)j * D + c], s);
        s = 0.5f * warp_sum(s);
        if (lane == 0) wrow[j] = (gate && s > ln_b) ? 0.f : s;
    }
}

}  // namespace pisa
