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
// score tree runs on scalar __fmul_rn / __fadd_rn only: packed fp32x2
// multiplies and adds were measured not to reproduce the separately rounded
// scalar results.
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

// Canonical score split over four lanes (one residue class mod 4 each).  The
// canonical tree (a[i] = a[i] + a[i + h], first level i < D/2 pairing the
// products of columns i and i + D/2, then h = D/4 .. 1) only ever adds two
// entries of the same residue mod 4 while h >= 4, so lane r (the entries
// i = r + 4m) runs those levels alone on its D/8 values; the last two levels
// (h = 2: a[0] + a[2], a[1] + a[3]; h = 1: a[0] + a[1]) are two shuffles.  Every
// product and sum is one IEEE fp32 round-to-nearest operation (__fmul_rn /
// __fadd_rn, never fused), so the score is the same bit for bit as the serial
// canonical order.  q holds q[r + 4m] (m < D/8) then q[D/2 + r + 4m]; k is the
// block's segment for residue r in the same order.  The result is valid in
// lane r = 0 of the group.  (Packed fp32x2 multiplies and adds do not
// reproduce separately rounded scalar operations, so they are not used.)
template <int D>
__device__ __forceinline__ float canonical_dot4(const float (&q)[D / 4], const float* __restrict__ k, int r) {
    constexpr int H = D / 8;
    float a[H];
    const float4* k4 = reinterpret_cast<const float4*>(k);
#pragma unroll
    for (int m = 0; m < H / 4; ++m) {
        const float4 lo = k4[m], hi = k4[H / 4 + m];
        a[4 * m + 0] = __fadd_rn(__fmul_rn(q[4 * m + 0], lo.x), __fmul_rn(q[H + 4 * m + 0], hi.x));
        a[4 * m + 1] = __fadd_rn(__fmul_rn(q[4 * m + 1], lo.y), __fmul_rn(q[H + 4 * m + 1], hi.y));
        a[4 * m + 2] = __fadd_rn(__fmul_rn(q[4 * m + 2], lo.z), __fmul_rn(q[H + 4 * m + 2], hi.z));
        a[4 * m + 3] = __fadd_rn(__fmul_rn(q[4 * m + 3], lo.w), __fmul_rn(q[H + 4 * m + 3], hi.w));
    }
    float v = tree_sum<H>(a);  // global levels h = D/4 .. 4: lane r now holds a[r]
    v = __fadd_rn(v, __shfl_down_sync(0xffffffffu, v, 2));  // h = 2 (lanes r = 0, 1)
    v = __fadd_rn(v, __shfl_down_sync(0xffffffffu, v, 1));  // h = 1 (lane r = 0)
    (void)r;
    return v;
}

// The K-th largest of the warp's ordered keys, NKT per lane (key j = lane + 32 i of the
// score row st, j < nblk; 0 < K < nblk): a binary search on the key's bits, from the
// highest bit in which the warp's smallest and largest keys differ (the bits above it
// are common to every key, so to the answer).  Sets `need` to how many of the keys equal
// to the result are taken (the lowest block indices first).
template <int NKT>
__device__ __forceinline__ uint32_t kth_ordered_key(const float* st, int nblk, int K, int& need) {
    const int lane = threadIdx.x & 31;
    uint32_t kv[NKT];
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int i = 0; i < NKT; ++i) {
        const int j = lane + 32 * i;
        kv[i] = j < nblk ? ordered_key(st[j]) : 0u;  // 0 sorts below every score
        if (j < nblk) {
            lo = min(lo, kv[i]);
            hi = max(hi, kv[i]);
        }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    uint32_t thr = hi;
    if (lo != hi) {
        const int top = 31 - __clz(lo ^ hi);  // highest differing bit
        thr = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
        for (int bit = top; bit >= 0; --bit) {
            const uint32_t cand = thr | (1u << bit);
            int cnt = 0;
#pragma unroll
            for (int i = 0; i < NKT; ++i) cnt += kv[i] >= cand;
            cnt = __reduce_add_sync(0xffffffffu, cnt);
            if (cnt >= K) thr = cand;
        }
    }
    int gt = 0;
#pragma unroll
    for (int i = 0; i < NKT; ++i) gt += kv[i] > thr;
    need = K - __reduce_add_sync(0xffffffffu, gt);
    return thr;
}

// Two canonical scores of the same tile at once (blocks ka and kb, each given as the
// lane's residue segment): the same operations as canonical_dot4, interleaved so that
// each lane has two independent chains in flight.
template <int D>
__device__ __forceinline__ void canonical_dot4x2(const float (&q)[D / 4], const float* __restrict__ ka,
                                                 const float* __restrict__ kb, float& sa, float& sb) {
    constexpr int H = D / 8;
    float a[H], b[H];
    const float4* ka4 = reinterpret_cast<const float4*>(ka);
    const float4* kb4 = reinterpret_cast<const float4*>(kb);
#pragma unroll
    for (int m = 0; m < H / 4; ++m) {
        const float4 alo = ka4[m], ahi = ka4[H / 4 + m];
        const float4 blo = kb4[m], bhi = kb4[H / 4 + m];
        a[4 * m + 0] = __fadd_rn(__fmul_rn(q[4 * m + 0], alo.x), __fmul_rn(q[H + 4 * m + 0], ahi.x));
        b[4 * m + 0] = __fadd_rn(__fmul_rn(q[4 * m + 0], blo.x), __fmul_rn(q[H + 4 * m + 0], bhi.x));
        a[4 * m + 1] = __fadd_rn(__fmul_rn(q[4 * m + 1], alo.y), __fmul_rn(q[H + 4 * m + 1], ahi.y));
        b[4 * m + 1] = __fadd_rn(__fmul_rn(q[4 * m + 1], blo.y), __fmul_rn(q[H + 4 * m + 1], bhi.y));
        a[4 * m + 2] = __fadd_rn(__fmul_rn(q[4 * m + 2], alo.z), __fmul_rn(q[H + 4 * m + 2], ahi.z));
        b[4 * m + 2] = __fadd_rn(__fmul_rn(q[4 * m + 2], blo.z), __fmul_rn(q[H + 4 * m + 2], bhi.z));
        a[4 * m + 3] = __fadd_rn(__fmul_rn(q[4 * m + 3], alo.w), __fmul_rn(q[H + 4 * m + 3], ahi.w));
        b[4 * m + 3] = __fadd_rn(__fmul_rn(q[4 * m + 3], blo.w), __fmul_rn(q[H + 4 * m + 3], bhi.w));
    }
#pragma unroll
    for (int h = H / 2; h >= 1; h >>= 1) {
#pragma unroll
        for (int i = 0; i < h; ++i) {
            a[i] = __fadd_rn(a[i], a[i + h]);
            b[i] = __fadd_rn(b[i], b[i + h]);
        }
    }
    float va = a[0], vb = b[0];
    const float pa = __shfl_down_sync(0xffffffffu, va, 2), pb = __shfl_down_sync(0xffffffffu, vb, 2);
    va = __fadd_rn(va, pa);  // h = 2
    vb = __fadd_rn(vb, pb);
    const float ra = __shfl_down_sync(0xffffffffu, va, 1), rb = __shfl_down_sync(0xffffffffu, vb, 1);
    sa = __fadd_rn(va, ra);  // h = 1
    sb = __fadd_rn(vb, rb);
}

template <int D>
struct SelectCfg {
    static constexpr int THREADS = 256;
    static constexpr int JC = 32;          // centroids staged per chunk
    static constexpr int SEG = D / 4 + 4;  // floats per residue segment of a staged centroid (padded)
};

// Query tiles per CTA: 16 (two groups of 8 tiles, four lanes a tile) when the score
// table leaves room for three CTAs per SM, else 8.
template <int D>
inline size_t select_smem_bytes(int QT, int nblk) {
    return sizeof(float) * ((size_t)QT * D + (size_t)SelectCfg<D>::JC * 4 * SelectCfg<D>::SEG +
                            (size_t)QT * (nblk + 1));
}
template <int D>
inline int select_tiles_per_cta(int nblk) {
    return select_smem_bytes<D>(16, nblk) <= 72 * 1024 ? 16 : 8;
}

// One CTA per (group of QT query tiles, bh), 8 warps.
//   1. canonical tile means (thread per (tile, column));
//   2. scores: lane 4 tl + r of a warp works on tile tl of the warp's tile group
//      and residue r of the canonical tree; the centroids are staged JC at a
//      time, each split into its four residue segments; the warps of a tile
//      group split the blocks of a chunk between them; with a routing bias
//      ([BH, nblk], or null) each score gets bias_j added;
//   3. top-K per tile (warp per tile): binary search for the K-th largest
//      ordered score, then ties broken by ascending block index with ballots;
//      the ballots are the mask words and give the ascending index list.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(256, 3) select_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                                                        int L, int nblk, int K, int words, int QT,
                                                        int32_t* __restrict__ idx, uint32_t* __restrict__ mask,
                                                        const float* __restrict__ bias,
                                                        float* __restrict__ scores_out) {
    using C = SelectCfg<D>;
    extern __shared__ __align__(16) float sm_sel[];
    float* qbar = sm_sel;                    // [QT][D]
    float* kst = qbar + QT * D;              // [JC][4][SEG]: residue segments of the staged centroids
    float* sc = kst + C::JC * 4 * C::SEG;    // [QT][nblk + 1]
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
    const int ngroups = QT / 8;            // tile groups of 8 tiles
    const int grp = warp % ngroups;        // this warp's tile group
    const int wsplit = 8 / ngroups;        // warps sharing a tile group (they split the blocks)
    const int wpart = warp / ngroups;
    const int tl = lane >> 2, r = lane & 3;
    const int t = grp * 8 + tl;            // tile of this lane inside the CTA
    const bool live = t < nq;
    float qr[D / 4];  // q[r + 4m], then q[D/2 + r + 4m]
    {
        const float* qt_ = qbar + (live ? t : 0) * D;
#pragma unroll
        for (int m = 0; m < D / 8; ++m) {
            qr[m] = qt_[r + 4 * m];
            qr[D / 8 + m] = qt_[D / 2 + r + 4 * m];
        }
    }
    const float4* kb4 = reinterpret_cast<const float4*>(kbar + (size_t)bh * nblk * D);
    for (int j0 = 0; j0 < nblk; j0 += C::JC) {
        const int nj = min(C::JC, nblk - j0);
        // stage the chunk split into residue segments: column i of block jj goes to
        // segment i % 4 at position (i % (D/2)) / 4 + (i >= D/2 ? D/8 : 0)
        for (int e = tid; e < nj * D / 4; e += C::THREADS) {
            const int jj = e / (D / 4), c4 = (e % (D / 4)) * 4;
            const float4 v = kb4[(size_t)j0 * D / 4 + e];
            const int pos = (c4 % (D / 2)) / 4 + (c4 >= D / 2 ? D / 8 : 0);
            float* seg = kst + (jj * 4) * C::SEG + pos;
            seg[0 * C::SEG] = v.x;
            seg[1 * C::SEG] = v.y;
            seg[2 * C::SEG] = v.z;
            seg[3 * C::SEG] = v.w;
        }
        __syncthreads();
        // two blocks per iteration (jj and jj + wsplit) for two independent chains a lane
        for (int jj = wpart; jj < nj; jj += 2 * wsplit) {
            const int jj2 = jj + wsplit;
            const bool two = jj2 < nj;
            float s, s2;
            canonical_dot4x2<D>(qr, kst + (jj * 4 + r) * C::SEG, kst + ((two ? jj2 : jj) * 4 + r) * C::SEG, s, s2);
            // covariance-aware routing: one fp32 add of the block's bias
            if (bias) {
                s = __fadd_rn(s, __ldg(bias + (size_t)bh * nblk + j0 + jj));
                if (two) s2 = __fadd_rn(s2, __ldg(bias + (size_t)bh * nblk + j0 + jj2));
            }
            if (live && r == 0) {
                sc[t * SS + j0 + jj] = s;
                if (two) sc[t * SS + j0 + jj2] = s2;
            }
        }
        __syncthreads();
    }

    // the score table itself, when asked for ([BH, nblk, nblk] fp32)
    if (scores_out) {
        for (int e = tid; e < nq * nblk; e += C::THREADS) {
            const int tt = e / nblk, jj = e % nblk;
            scores_out[((size_t)bh * nblk + i0 + tt) * nblk + jj] = sc[tt * SS + jj];
        }
    }

    // 3. top-K, one warp per tile.  For nblk <= 1024 every lane keeps its
    // blocks' ordered keys (j = lane + 32 i) in registers during the search
    // (kth_ordered_key); longer rows are searched from shared memory.
    const unsigned lt_mask = (1u << lane) - 1u;
    const int nk = (nblk + 31) / 32;
    for (int tt = warp; tt < nq; tt += 8) {
        const float* st = sc + tt * SS;
        const size_t row = (size_t)bh * nblk + i0 + tt;
        uint32_t thr = 0u;  // K-th largest ordered score (unused when K is 0 or nblk)
        int need = 0;       // how many of the ties at thr to take, lowest index first
        if (K > 0 && K < nblk) {
            if (nk <= 32) {
                // every lane keeps its blocks' ordered keys in registers during the search
                if (nk <= 4)
                    thr = kth_ordered_key<4>(st, nblk, K, need);
                else if (nk <= 8)
                    thr = kth_ordered_key<8>(st, nblk, K, need);
                else if (nk <= 16)
                    thr = kth_ordered_key<16>(st, nblk, K, need);
                else
                    thr = kth_ordered_key<32>(st, nblk, K, need);
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