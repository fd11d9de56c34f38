// Block selection: tile-mean query against every key centroid, top-K blocks.
//
// PISA paper, section 3.2 "Formulation" (query blocks share one selected set
// S_i) and Figure 3 caption (block means of queries and keys, block-wise
// top-K); the score is the MoBA-style centroid product of the "Sparse Linear
// Attention" blog, section "Sparse Attention".  Eq. 7's softmax is monotone and
// is not applied.  Ties go to the lower block index.
//
// Every fp32 operation follows the canonical order of the C ABI comment:
// tile means by the pairwise tree over the B rows, scores by the pairwise
// tree over the d products, each product and sum rounded on its own.
#pragma once

#include "common.cuh"

namespace pisa {

// Order-preserving map of an fp32 score to uint32 (larger score -> larger
// key); +0 and -0 map to the same key.
__device__ __forceinline__ uint32_t ordered_key(float s) {
    uint32_t u = __float_as_uint(s);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One CTA per (query tile, bh); 256 threads.  P = power of two >= nblk.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(256) select_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                                                     int L, int nblk, int K, int words, int P,
                                                     int32_t* __restrict__ idx, uint32_t* __restrict__ mask) {
    extern __shared__ __align__(16) unsigned long long sm_sel[];
    unsigned long long* keys = sm_sel;                      // [P]
    float* qbar = (float*)(keys + P);                       // [D]
    uint32_t* mw = (uint32_t*)(qbar + D);                   // [words]
    uint32_t* off = mw + words;                             // [words]
    const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;

    // 1. canonical tile mean, thread c owns column c
    if (tid < D) {
        const T* src = q + ((size_t)bh * L + (size_t)i * BS) * D + tid;
        float a[BS];
#pragma unroll
        for (int n = 0; n < BS; ++n) a[n] = to_f(src[(size_t)n * D]);
        qbar[tid] = __fmul_rn(tree_sum<BS>(a), 1.0f / (float)BS);
    }
    for (int e = tid; e < words; e += 256) mw[e] = 0u;
    __syncthreads();

    // 2. scores, one warp per block j; lane holds columns lane + 32*w
    constexpr int W = D / 32;
    float qv[W];
#pragma unroll
    for (int w = 0; w < W; ++w) qv[w] = qbar[lane + 32 * w];
    const float* kb = kbar + (size_t)bh * nblk * D;
    for (int j = warp; j < P; j += 8) {
        if (j >= nblk) {
            if (lane == 0) keys[j] = 0ull;
            continue;
        }
        float p[W];
#pragma unroll
        for (int w = 0; w < W; ++w) p[w] = __fmul_rn(qv[w], kb[(size_t)j * D + lane + 32 * w]);
        // tree levels h = D/2 .. 32 inside the lane, h = 16 .. 1 across lanes
#pragma unroll
        for (int h = W / 2; h >= 1; h >>= 1) {
#pragma unroll
            for (int w = 0; w < h; ++w) p[w] = __fadd_rn(p[w], p[w + h]);
        }
        float s = p[0];
#pragma unroll
        for (int h = 16; h >= 1; h >>= 1) s = __fadd_rn(s, __shfl_down_sync(0xffffffffu, s, h));
        if (lane == 0) keys[j] = ((unsigned long long)ordered_key(s) << 32) | (0xffffffffu - (uint32_t)j);
    }
    __syncthreads();

    // 3. bitonic sort, descending
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = tid; t < P / 2; t += 256) {
                const int lo = 2 * stride * (t / stride) + (t % stride);
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long a = keys[lo], b = keys[hi];
                if ((a < b) == desc) {
                    keys[lo] = b;
                    keys[hi] = a;
                }
            }
            __syncthreads();
        }
    }

    // 4. mask of the first K, then the ascending index list
    for (int t = tid; t < K; t += 256) {
        const uint32_t j = 0xffffffffu - (uint32_t)(keys[t] & 0xffffffffull);
        atomicOr(&mw[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t acc = 0;
        for (int w = 0; w < words; ++w) {
            off[w] = acc;
            acc += __popc(mw[w]);
        }
    }
    __syncthreads();
    const size_t row = (size_t)bh * nblk + i;
    for (int w = tid; w < words; w += 256) {
        const uint32_t bits = mw[w];
        if (mask) mask[row * words + w] = bits;
        if (idx) {
            uint32_t b = bits, o = off[w];
            while (b) {
                const int t = __ffs(b) - 1;
                idx[row * K + o++] = w * 32 + t;
                b &= b - 1;
            }
        }
    }
}

}  // namespace pisa
