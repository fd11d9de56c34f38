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
// tree over the d products, each product and sum rounded on its own.  The
// score tree runs on packed fp32x2 operations (two independent IEEE
// round-to-nearest operations each), which leaves every rounding unchanged.
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

__device__ __forceinline__ unsigned long long f2_pack(float2 v) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
    return r;
}
__device__ __forceinline__ float2 f2_unpack(unsigned long long r) {
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Canonical score: p_c = q_c * k_c rounded, then the pairwise tree
// a[i] = a[i] + a[i + h], h = D/2 .. 1.  Lanes of packed pairs hold
// (a[2m], a[2m+1]); every level with h >= 2 pairs up element-wise.
template <int D>
__device__ __forceinline__ float canonical_dot(const unsigned long long (&q2)[D / 2], const float* __restrict__ k) {
    unsigned long long a[D / 4];
    const float4* k4 = reinterpret_cast<const float4*>(k);
#pragma unroll
    for (int m = 0; m < D / 4; m += 2) {
        // products of columns 2m .. 2m+3 and of D/2 + 2m .. D/2 + 2m + 3
        const float4 lo = k4[m / 2], hi = k4[(D / 2 + 2 * m) / 4];
        const unsigned long long plo0 = f2_mul(q2[m], f2_pack(make_float2(lo.x, lo.y)));
        const unsigned long long plo1 = f2_mul(q2[m + 1], f2_pack(make_float2(lo.z, lo.w)));
        const unsigned long long phi0 = f2_mul(q2[D / 4 + m], f2_pack(make_float2(hi.x, hi.y)));
        const unsigned long long phi1 = f2_mul(q2[D / 4 + m + 1], f2_pack(make_float2(hi.z, hi.w)));
        a[m] = f2_add(plo0, phi0);
        a[m + 1] = f2_add(plo1, phi1);
    }
#pragma unroll
    for (int h = D / 8; h >= 1; h >>= 1) {
#pragma unroll
        for (int m = 0; m < h; ++m) a[m] = f2_add(a[m], a[m + h]);
    }
    const float2 last = f2_unpack(a[0]);
    return __fadd_rn(last.x, last.y);
}

template <int D>
struct SelectCfg {
    static constexpr int THREADS = 256;
    static constexpr int JC = 64;  // centroids staged per chunk
};

// Query tiles per CTA (one per lane of a warp, at most 32) so that the score
// table fits next to the staged tile means and centroids.
template <int D>
inline int select_tiles_per_cta(int nblk) {
    const long budget = 200 * 1024 - (long)sizeof(float) * (32 * D + SelectCfg<D>::JC * D);
    long qt = budget / ((long)sizeof(float) * (nblk + 1));
    return (int)(qt > 32 ? 32 : (qt < 1 ? 1 : qt));
}

template <int D>
inline size_t select_smem_bytes(int QT, int nblk) {
    return sizeof(float) * ((size_t)QT * D + (size_t)SelectCfg<D>::JC * D + (size_t)QT * (nblk + 1));
}

// One CTA per (group of QT query tiles, bh), 8 warps.
//   1. canonical tile means (thread per (tile, column));
//   2. scores: lane t of every warp holds tile t's mean in registers, the
//      centroids are staged JC at a time and read as broadcasts; warp w takes
//      the blocks jj = w, w+8, ... of each chunk;
//   3. top-K per tile (warp per tile): binary search for the K-th largest
//      ordered score, then ties broken by ascending block index with ballots;
//      the ballots are the mask words and give the ascending index list.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(256, 1) select_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                                                        int L, int nblk, int K, int words, int QT,
                                                        int32_t* __restrict__ idx, uint32_t* __restrict__ mask) {
    using C = SelectCfg<D>;
    extern __shared__ __align__(16) float sm_sel[];
    float* qbar = sm_sel;                 // [QT][D]
    float* kst = qbar + QT * D;           // [JC][D]
    float* sc = kst + C::JC * D;          // [QT][nblk + 1]
    const int SS = nblk + 1;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32, bh = blockIdx.y;
    const int i0 = blockIdx.x * QT;
    const int nq = min(QT, nblk - i0);

    // 1. tile means; bf16 tiles of 64 rows are read as bf16x2 pairs (two
    // columns per thread) so that more bytes are in flight per thread
    constexpr int VEC = (sizeof(T) == 2 && BS <= 64) ? 2 : 1;
    constexpr int CPT = D / VEC;  // threads per tile
    for (int e = tid; e < nq * CPT; e += C::THREADS) {
        const int t = e / CPT, c = (e % CPT) * VEC;
        const T* src = q + ((size_t)bh * L + (size_t)(i0 + t) * BS) * D + c;
        if constexpr (VEC == 2) {
            float a0[BS], a1[BS];
#pragma unroll
            for (int n = 0; n < BS; ++n) {
                const __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(src + (size_t)n * D);
                a0[n] = __low2float(p);
                a1[n] = __high2float(p);
            }
            qbar[t * D + c] = __fmul_rn(tree_sum<BS>(a0), 1.0f / (float)BS);
            qbar[t * D + c + 1] = __fmul_rn(tree_sum<BS>(a1), 1.0f / (float)BS);
        } else {
            float a[BS];
#pragma unroll
            for (int n = 0; n < BS; ++n) a[n] = to_f(src[(size_t)n * D]);
            qbar[t * D + c] = __fmul_rn(tree_sum<BS>(a), 1.0f / (float)BS);
        }
    }
    __syncthreads();

    // 2. scores
    const bool live = lane < nq;
    unsigned long long q2[D / 2];
    {
        const float2* qs = reinterpret_cast<const float2*>(qbar + (live ? lane : 0) * D);
#pragma unroll
        for (int m = 0; m < D / 2; ++m) q2[m] = f2_pack(qs[m]);
    }
    const float4* kb4 = reinterpret_cast<const float4*>(kbar + (size_t)bh * nblk * D);
    for (int j0 = 0; j0 < nblk; j0 += C::JC) {
        const int nj = min(C::JC, nblk - j0);
        float4* kst4 = reinterpret_cast<float4*>(kst);
        for (int e = tid; e < nj * D / 4; e += C::THREADS) kst4[e] = kb4[(size_t)j0 * D / 4 + e];
        __syncthreads();
        for (int jj = warp; jj < nj; jj += 8) {
            const float s = canonical_dot<D>(q2, kst + jj * D);
            if (live) sc[lane * SS + j0 + jj] = s;
        }
        __syncthreads();
    }

    // 3. top-K, one warp per tile.  For nblk <= 1024 every lane keeps its
    // blocks' ordered keys (j = lane + 32 i) in registers during the search.
    const unsigned lt_mask = (1u << lane) - 1u;
    const int nk = (nblk + 31) / 32;
    for (int t = warp; t < nq; t += 8) {
        const float* st = sc + t * SS;
        const size_t row = (size_t)bh * nblk + i0 + t;
        uint32_t thr = 0u;  // K-th largest ordered score (unused when K is 0 or nblk)
        int need = 0;       // how many of the ties at thr to take, lowest index first
        if (K > 0 && K < nblk) {
            if (nk <= 32) {
                uint32_t kv[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int j = lane + 32 * i;
                    kv[i] = (i < nk && j < nblk) ? ordered_key(st[j]) : 0u;  // 0 sorts below every score
                }
                for (int bit = 31; bit >= 0; --bit) {
                    const uint32_t cand = thr | (1u << bit);
                    int cnt = 0;
#pragma unroll
                    for (int i = 0; i < 32; ++i) cnt += (i < nk) & (kv[i] >= cand);
                    cnt = __reduce_add_sync(0xffffffffu, cnt);
                    if (cnt >= K) thr = cand;
                }
                int gt = 0;
#pragma unroll
                for (int i = 0; i < 32; ++i) gt += (i < nk) & (kv[i] > thr);
                need = K - __reduce_add_sync(0xffffffffu, gt);
            } else {
                for (int bit = 31; bit >= 0; --bit) {
                    const uint32_t cand = thr | (1u << bit);
                    int cnt = 0;
                    for (int j = lane; j < nblk; j += 32) cnt += ordered_key(st[j]) >= cand;
                    cnt = __reduce_add_sync(0xffffffffu, cnt);
                    if (cnt >= K) thr = cand;
                }
                int gt = 0;
                for (int j = lane; j < nblk; j += 32) gt += ordered_key(st[j]) > thr;
                need = K - __reduce_add_sync(0xffffffffu, gt);
            }
        }
        int off = 0, eq_seen = 0;
        for (int w = 0; w < words; ++w) {
            // every lane takes part in every ballot; lanes past nblk vote "no"
            const int j = w * 32 + lane;
            const bool in = j < nblk;
            const uint32_t o = in ? ordered_key(st[j]) : 0u;
            const unsigned eq = __ballot_sync(0xffffffffu, in && o == thr);
            const int rank = eq_seen + __popc(eq & lt_mask);
            eq_seen += __popc(eq);
            const bool sel = in && (K == nblk || (K > 0 && (o > thr || (o == thr && rank < need))));
            const unsigned bits = __ballot_sync(0xffffffffu, sel);
            if (mask && lane == 0) mask[row * words + w] = bits;
            if (idx && sel) idx[row * K + off + __popc(bits & lt_mask)] = j;
            off += __popc(bits);
        }
    }
}

}  // namespace pisa
