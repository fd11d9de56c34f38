// Backward pass of the piecewise sparse attention: dq, dk, dv of sum_t dO_t . o_t.
//
// The pages define only the forward: PISA paper section 3.2 "Formulation" (o_t,
// D_t) and Figure 3; "Sparse Linear Attention" blog, the sparse-linear and PWT
// sections (the virtual token, H_j, w_tj and the ln B gate).  These gradients
// differentiate that forward with the block selection held fixed, and for order
// 2 the gate decision too; the PWT blog trains with the routing detached in the
// same way.
//
// Per query row t (x_n = q_t.k_n, G_n = dO_t.v_n, delta = dO_t.o_t, m and D the
// shared max and denominator of the forward):
//   selected key n           P_n = e^{x_n - m} / D,      dS_n = P_n (G_n - delta)
//   key n of unselected j    sb = q_t.kbar_j = mean of x over the block, u_n = x_n - sb,
//                            l = sb + w (w = [order 2] sum u^2 / 2B, zeroed by the gate),
//                            a = e^{l - m} / D,           P_n = a (1 + c1 u_n),
//                            inner = sum_n G_n (1 + c1 u_n) - B delta,
//                            dS_n = a (dl_n inner + c1 (G_n - mean G)),
//                            dl_n = 1/B (+ u_n / B for order 2 with the gate open)
//   dq_t = sum_n dS_tn k_n,   dk_n = sum_t dS_tn q_t,   dv_n = sum_t P_tn dO_t
// (c1 = 1 for order >= 1, 0 for order 0).
//
// Three kernels.  Each recomputes S = Q K^T (and G = dO V^T) tile by tile
// instead of storing L^2 values:
//   bwd_rowstat_kernel  per row: m, D and delta (one 64-row tile per CTA);
//   bwd_dq_kernel       query-major: one 64-row tile per CTA, looping over the
//                       key blocks;
//   bwd_dkdv_kernel     key-major: one key block per CTA, looping over 32-row
//                       query chunks.
// Every reduction over a block (sb, sum G, sum G u, the spread behind w) runs
// over the B keys of one block, which is one tile of these kernels, so no
// per-(row, block) value crosses kernels.
//
// Tile products: bf16 inputs use warp-level mma.sync m16n8k16 (bf16 operands,
// fp32 accumulators) with operands gathered by ldmatrix (.trans for the
// k-major ones).  fp32 inputs use the same accumulator fragment layout,
// computed with fp32 FMAs on the CUDA cores (the reference-precision variant).
// Global tiles move with cp.async: double-buffered for bf16 (the next key
// block or query chunk loads while this one is computed), one stage for fp32
// (two do not fit in shared memory).  No kernel here waits on a flag; the
// only waits are __syncthreads and cp.async.wait_group on the thread's own
// copies.
#pragma once

#include <math.h>

#include "common.cuh"

namespace pisa {
namespace bwd {

constexpr int kQT = 64;   // rows per CTA of the row-statistics and dq kernels (4 warps x 16)
constexpr int kQC = 32;   // query rows per step of the dk/dv kernel
constexpr int kPad = 8;   // elements of padding per shared-memory row (conflict-free fragment loads)

template <typename T, int D, int BS>
struct Cfg {
    static constexpr int NST = sizeof(T) == 2 ? 2 : 1;  // cp.async stages of the streamed tiles
    static constexpr int LD = D + kPad;     // q, k, v, dO tiles
    static constexpr int LDS = BS + kPad;   // dS tile of the dq kernel
    static constexpr int LDP = kQC + kPad;  // P^T and dS^T tiles of the dk/dv kernel
    static constexpr int NW_KV = BS / 16;   // warps of the dk/dv kernel (16 keys each)
    static constexpr size_t ROWSTAT_SMEM = sizeof(T) * (size_t)(kQT + NST * BS) * LD;
    // dq kernel: Q, dO, then NST stages of (K, V); dS reuses the current stage's V space
    static constexpr size_t DQ_SMEM = sizeof(T) * (size_t)(2 * kQT + 2 * NST * BS) * LD;
    // dk/dv kernel: K, V, NST stages of (Q, dO), P^T, dS^T; then fp32 scratch and NST stages
    // of the chunk's m, 1/D, delta
    static constexpr size_t DKDV_T = (size_t)(2 * BS + 2 * NST * kQC) * LD + 2 * (size_t)BS * LDP;
    static constexpr size_t DKDV_SMEM =
        sizeof(T) * DKDV_T + sizeof(float) * ((size_t)NW_KV * kQC * 4 + 3 * NST * kQC);
    static_assert(kQT * LDS <= BS * LD, "dS tile must fit in the V tile");
    static_assert((sizeof(T) * DKDV_T) % 16 == 0, "float scratch must stay aligned");
    static_assert((NW_KV * kQC * 4 * sizeof(float)) % 16 == 0, "row statistics must stay 16-byte aligned");
};

// ---------------------------------------------------------------------------
// warp-level tile products: acc[nt] (16 x 8 each) += A[16 x KD] * B[KD x 8 NT]
// Accumulator fragment (mma m16n8 layout), lane = 4 g + t:
//   acc[nt][0..1] = C[g][8 nt + 2t + {0,1}],  acc[nt][2..3] = C[g + 8][8 nt + 2t + {0,1}]
// A is row-major in shared memory (row stride lda elements).
// "nk" form: B[k][n] = Bn[n * ldb + k];  "kn" form: B[k][n] = Bk[k * ldb + n].
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ldmatrix x4: lanes 8m .. 8m+7 give the row addresses of 8 x 8 matrix m (16-byte rows);
// register m of lane 4g + t receives row g, columns 2t and 2t+1 of matrix m (.trans: row 2t
// and 2t+1 of column g), low half = first element.
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], const bf16* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr(p))
                 : "memory");
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], const bf16* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr(p))
                 : "memory");
}

// A fragment of the 16 x 16 slice at column k0: registers (row g, k0+2t..), (row g+8, k0+2t..),
// (row g, k0+8+2t..), (row g+8, k0+8+2t..) = matrices (rows 0-7 | 8-15) x (cols k0 | k0+8).
__device__ __forceinline__ void load_a(uint32_t (&a)[4], const bf16* A, int lda, int k0, int lane) {
    const int m = lane >> 3, r = lane & 7;
    ldsm4(a, A + ((m & 1) * 8 + r) * lda + k0 + (m >> 1) * 8);
}

// NT even.  B fragments of n-tiles nt and nt+1 in one ldmatrix: (b0, b1) of tile nt, then of nt+1;
// b0 = (k0+2t.., n = 8nt+g), b1 = (k0+8+2t.., n).
template <int NT, int KD>
__device__ __forceinline__ void warp_mma_nk(float (&acc)[NT][4], const bf16* A, int lda, const bf16* Bn, int ldb,
                                            int lane) {
    const int m = lane >> 3, r = lane & 7;
#pragma unroll
    for (int k0 = 0; k0 < KD; k0 += 16) {
        uint32_t a[4];
        load_a(a, A, lda, k0, lane);
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
            uint32_t b[4];  // Bn rows are n: matrices (n-tile nt | nt+1) x (cols k0 | k0+8)
            ldsm4(b, Bn + ((nt + (m >> 1)) * 8 + r) * ldb + k0 + (m & 1) * 8);
            mma16816(acc[nt], a, b[0], b[1]);
            mma16816(acc[nt + 1], a, b[2], b[3]);
        }
    }
}

template <int NT, int KD>
__device__ __forceinline__ void warp_mma_kn(float (&acc)[NT][4], const bf16* A, int lda, const bf16* Bk, int ldb,
                                            int lane) {
    const int m = lane >> 3, r = lane & 7;
#pragma unroll
    for (int k0 = 0; k0 < KD; k0 += 16) {
        uint32_t a[4];
        load_a(a, A, lda, k0, lane);
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
            uint32_t b[4];  // Bk rows are k: matrices (rows k0 | k0+8) x (n-tile nt | nt+1), transposed
            ldsm4t(b, Bk + (k0 + (m & 1) * 8 + r) * ldb + (nt + (m >> 1)) * 8);
            mma16816(acc[nt], a, b[0], b[1]);
            mma16816(acc[nt + 1], a, b[2], b[3]);
        }
    }
}

// Two nk products of the same shape in one k loop (acc1 += A1 B1, acc2 += A2 B2): twice the
// independent accumulator chains; every accumulator sees the same operations in the same order
// as in two separate calls.
template <int NT, int KD>
__device__ __forceinline__ void warp_mma_nk2(float (&acc1)[NT][4], const bf16* A1, const bf16* B1,
                                             float (&acc2)[NT][4], const bf16* A2, const bf16* B2, int lda,
                                             int ldb, int lane) {
    const int m = lane >> 3, r = lane & 7;
#pragma unroll
    for (int k0 = 0; k0 < KD; k0 += 16) {
        uint32_t a1[4], a2[4];
        load_a(a1, A1, lda, k0, lane);
        load_a(a2, A2, lda, k0, lane);
#pragma unroll
        for (int nt = 0; nt < NT; nt += 2) {
            uint32_t b1[4], b2[4];
            const int off = ((nt + (m >> 1)) * 8 + r) * ldb + k0 + (m & 1) * 8;
            ldsm4(b1, B1 + off);
            ldsm4(b2, B2 + off);
            mma16816(acc1[nt], a1, b1[0], b1[1]);
            mma16816(acc2[nt], a2, b2[0], b2[1]);
            mma16816(acc1[nt + 1], a1, b1[2], b1[3]);
            mma16816(acc2[nt + 1], a2, b2[2], b2[3]);
        }
    }
}

// fp32 operands: the same accumulator fragment, fp32 FMAs in k order.
template <int NT, int KD>
__device__ __forceinline__ void warp_mma_nk(float (&acc)[NT][4], const float* A, int lda, const float* Bn, int ldb,
                                            int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int k = 0; k < KD; ++k) {
        const float a0 = A[g * lda + k], a1 = A[(g + 8) * lda + k];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float b0 = Bn[(nt * 8 + 2 * t) * ldb + k], b1 = Bn[(nt * 8 + 2 * t + 1) * ldb + k];
            acc[nt][0] = fmaf(a0, b0, acc[nt][0]);
            acc[nt][1] = fmaf(a0, b1, acc[nt][1]);
            acc[nt][2] = fmaf(a1, b0, acc[nt][2]);
            acc[nt][3] = fmaf(a1, b1, acc[nt][3]);
        }
    }
}

template <int NT, int KD>
__device__ __forceinline__ void warp_mma_kn(float (&acc)[NT][4], const float* A, int lda, const float* Bk, int ldb,
                                            int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int k = 0; k < KD; ++k) {
        const float a0 = A[g * lda + k], a1 = A[(g + 8) * lda + k];
        const float* r = Bk + k * ldb + 2 * t;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float b0 = r[nt * 8], b1 = r[nt * 8 + 1];
            acc[nt][0] = fmaf(a0, b0, acc[nt][0]);
            acc[nt][1] = fmaf(a0, b1, acc[nt][1]);
            acc[nt][2] = fmaf(a1, b0, acc[nt][2]);
            acc[nt][3] = fmaf(a1, b1, acc[nt][3]);
        }
    }
}

template <int NT, int KD>
__device__ __forceinline__ void warp_mma_nk2(float (&acc1)[NT][4], const float* A1, const float* B1,
                                             float (&acc2)[NT][4], const float* A2, const float* B2, int lda,
                                             int ldb, int lane) {
    warp_mma_nk<NT, KD>(acc1, A1, lda, B1, ldb, lane);
    warp_mma_nk<NT, KD>(acc2, A2, lda, B2, ldb, lane);
}

// two adjacent elements (columns c, c+1) of a staged operand tile in one store
__device__ __forceinline__ void st_pair(bf16* p, float x0, float x1) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(x0, x1);
}
__device__ __forceinline__ void st_pair(float* p, float x0, float x1) {
    *reinterpret_cast<float2*>(p) = make_float2(x0, x1);
}

template <int NT>
__device__ __forceinline__ void zero(float (&acc)[NT][4]) {
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
}

// sum / max over the 4 lanes of a quad (the lanes holding one accumulator row)
__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x + __shfl_xor_sync(0xffffffffu, x, 2);
}
__device__ __forceinline__ float quad_max(float x) {
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
    return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
// sum over the 8 lanes g = 0..7 with the same t (the lanes holding one accumulator column)
__device__ __forceinline__ float col_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    return x + __shfl_xor_sync(0xffffffffu, x, 16);
}

// rows x COLS elements from global (row-major, COLS contiguous) into shared memory of row stride ld,
// as 16-byte cp.async copies (the caller commits and waits)
template <typename T, int COLS>
__device__ __forceinline__ void cp_rows(T* dst, int ld, const T* __restrict__ src, int rows, int tid, int nthr) {
    constexpr int V = 16 / (int)sizeof(T);
    constexpr int PR = COLS / V;
    for (int e = tid; e < rows * PR; e += nthr) {
        const int r = e / PR, c = (e - r * PR) * V;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(saddr(dst + r * ld + c)),
                     "l"(src + (size_t)r * COLS + c)
                     : "memory");
    }
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

__device__ __forceinline__ bool selected(const uint32_t* __restrict__ mrow, int j) {
    return (__ldg(mrow + (j >> 5)) >> (j & 31)) & 1u;
}

// ---------------------------------------------------------------------------
// Row statistics: m_t and 1/D_t as the forward forms them (one shared max and
// one denominator over the exact selected keys and the B-weighted virtual
// tokens e^{l_tj} of the unselected blocks), and delta_t = dO_t . o_t.
// ---------------------------------------------------------------------------
template <typename T, int D, int BS>
__global__ void __launch_bounds__(128) bwd_rowstat_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ o, const T* __restrict__ dO,
                                                          const uint32_t* __restrict__ mask, int L, int nblk,
                                                          int words, int order, int gate, float* __restrict__ m_out,
                                                          float* __restrict__ dinv_out,
                                                          float* __restrict__ delta_out) {
    using C = Cfg<T, D, BS>;
    extern __shared__ __align__(16) unsigned char sm_bwd[];
    T* Qs = reinterpret_cast<T*>(sm_bwd);
    T* Kst = Qs + kQT * C::LD;  // NST stages of K_j
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2;
    const int bh = blockIdx.y, row0 = blockIdx.x * kQT;
    const size_t hoff = (size_t)bh * L * D;
    cp_rows<T, D>(Qs, C::LD, q + hoff + (size_t)row0 * D, kQT, tid, 128);
    if (C::NST == 2) cp_rows<T, D>(Kst, C::LD, k + hoff, BS, tid, 128);
    cp_commit();
    for (int r = warp * 16; r < warp * 16 + 16; ++r) {
        const size_t off = hoff + (size_t)(row0 + r) * D;
        float s = 0.f;
        for (int c = lane; c < D; c += 32) s = fmaf(to_f(dO[off + c]), to_f(o[off + c]), s);
        s = warp_sum(s);
        if (lane == 0) delta_out[(size_t)bh * L + row0 + r] = s;
    }
    const uint32_t* mrow = mask + ((size_t)bh * nblk + row0 / BS) * words;
    const float inv_b = 1.f / (float)BS, ln_b = logf((float)BS);
    float m[2] = {-INFINITY, -INFINITY}, den[2] = {0.f, 0.f};
#pragma unroll 1
    for (int j = 0; j < nblk; ++j) {
        if (C::NST == 1) {
            __syncthreads();  // K_{j-1} no longer read
            cp_rows<T, D>(Kst, C::LD, k + hoff + (size_t)j * BS * D, BS, tid, 128);
            cp_commit();
        }
        cp_wait_all();
        __syncthreads();  // K_j visible to all; every warp has finished block j-1
        if (C::NST == 2 && j + 1 < nblk) {
            cp_rows<T, D>(Kst + ((j + 1) & 1) * BS * C::LD, C::LD, k + hoff + (size_t)(j + 1) * BS * D, BS, tid,
                          128);
            cp_commit();
        }
        const T* Ks = Kst + (C::NST == 2 ? (j & 1) : 0) * BS * C::LD;
        float s[BS / 8][4];
        zero(s);
        warp_mma_nk<BS / 8, D>(s, Qs + warp * 16 * C::LD, C::LD, Ks, C::LD, lane);
        const bool sel = selected(mrow, j);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float mn, add;
            if (sel) {
                float bm = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < BS / 8; ++nt) bm = fmaxf(bm, fmaxf(s[nt][2 * h], s[nt][2 * h + 1]));
                mn = fmaxf(m[h], quad_max(bm));
                float se = 0.f;
#pragma unroll
                for (int nt = 0; nt < BS / 8; ++nt) se += expf(s[nt][2 * h] - mn) + expf(s[nt][2 * h + 1] - mn);
                add = quad_sum(se);
            } else {
                float sx = 0.f;
#pragma unroll
                for (int nt = 0; nt < BS / 8; ++nt) sx += s[nt][2 * h] + s[nt][2 * h + 1];
                const float sb = quad_sum(sx) * inv_b;
                float w = 0.f;
                if (order == 2) {
                    float sv = 0.f;
#pragma unroll
                    for (int nt = 0; nt < BS / 8; ++nt) {
                        const float u0 = s[nt][2 * h] - sb, u1 = s[nt][2 * h + 1] - sb;
                        sv = fmaf(u0, u0, fmaf(u1, u1, sv));
                    }
                    w = quad_sum(sv) * (0.5f * inv_b);
                    if (gate && w > ln_b) w = 0.f;
                }
                const float l = sb + w;
                mn = fmaxf(m[h], l);
                add = (float)BS * expf(l - mn);
            }
            den[h] = den[h] * expf(m[h] - mn) + add;
            m[h] = mn;
        }
    }
    if ((lane & 3) == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const size_t r = (size_t)bh * L + row0 + warp * 16 + g + 8 * h;
            m_out[r] = m[h];
            dinv_out[r] = 1.f / den[h];
        }
    }
}

// dS of the rows g + 8h of a warp's 16 x (8 NS) tile in place of S (row form: a
// row's B keys lie in one quad), for the query tile's selected/unselected block.
template <int NS, int BS>
__device__ __forceinline__ void row_grad(float (&s)[NS][4], const float (&gg)[NS][4], bool sel, int order, int gate,
                                         const float (&mr)[2], const float (&dinv)[2], const float (&del)[2]) {
    const float inv_b = 1.f / (float)BS, ln_b = logf((float)BS);
    const float c1 = order >= 1 ? 1.f : 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (sel) {
#pragma unroll
            for (int nt = 0; nt < NS; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float p = expf(s[nt][2 * h + e] - mr[h]) * dinv[h];
                    s[nt][2 * h + e] = p * (gg[nt][2 * h + e] - del[h]);
                }
        } else {
            float sx = 0.f, sg = 0.f;
#pragma unroll
            for (int nt = 0; nt < NS; ++nt) {
                sx += s[nt][2 * h] + s[nt][2 * h + 1];
                sg += gg[nt][2 * h] + gg[nt][2 * h + 1];
            }
            const float sb = quad_sum(sx) * inv_b;
            sg = quad_sum(sg);
            float sgu = 0.f, sv = 0.f;
#pragma unroll
            for (int nt = 0; nt < NS; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float u = s[nt][2 * h + e] - sb;
                    sgu = fmaf(gg[nt][2 * h + e], u, sgu);
                    sv = fmaf(u, u, sv);
                }
            sgu = quad_sum(sgu);
            sv = quad_sum(sv);
            float w = 0.f, q2 = 0.f;
            if (order == 2) {
                w = sv * (0.5f * inv_b);
                if (gate && w > ln_b) w = 0.f;
                else q2 = inv_b;
            }
            const float a = expf(sb + w - mr[h]) * dinv[h];
            const float inner = sg + c1 * sgu - (float)BS * del[h];
            const float gbar = sg * inv_b;
#pragma unroll
            for (int nt = 0; nt < NS; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float u = s[nt][2 * h + e] - sb;
                    s[nt][2 * h + e] = a * ((inv_b + q2 * u) * inner + c1 * (gg[nt][2 * h + e] - gbar));
                }
        }
    }
}

// ---------------------------------------------------------------------------
// dq: query-major.  Per key block: S = Q K_j^T and G = dO V_j^T for the
// warp's 16 rows, dS in registers (block reductions over the row's quad),
// then dq += dS K_j.  K_{j+1}, V_{j+1} load (cp.async) during block j.
// ---------------------------------------------------------------------------
template <typename T, int D, int BS>
__global__ void __launch_bounds__(128) bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                     const T* __restrict__ v, const T* __restrict__ dO,
                                                     const uint32_t* __restrict__ mask, int L, int nblk, int words,
                                                     int order, int gate, const float* __restrict__ mstat,
                                                     const float* __restrict__ dinvstat,
                                                     const float* __restrict__ delta, float* __restrict__ dq) {
    using C = Cfg<T, D, BS>;
    constexpr int NS = BS / 8, ND = D / 8;
    extern __shared__ __align__(16) unsigned char sm_bwd[];
    T* Qs = reinterpret_cast<T*>(sm_bwd);
    T* dOs = Qs + kQT * C::LD;
    T* KV = dOs + kQT * C::LD;  // NST stages of (K_j, V_j)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int bh = blockIdx.y, row0 = blockIdx.x * kQT;
    const size_t hoff = (size_t)bh * L * D;
    auto stage_kv = [&](int j, int st) {
        T* ks = KV + st * 2 * BS * C::LD;
        cp_rows<T, D>(ks, C::LD, k + hoff + (size_t)j * BS * D, BS, tid, 128);
        cp_rows<T, D>(ks + BS * C::LD, C::LD, v + hoff + (size_t)j * BS * D, BS, tid, 128);
    };
    cp_rows<T, D>(Qs, C::LD, q + hoff + (size_t)row0 * D, kQT, tid, 128);
    cp_rows<T, D>(dOs, C::LD, dO + hoff + (size_t)row0 * D, kQT, tid, 128);
    if (C::NST == 2) stage_kv(0, 0);
    cp_commit();
    float mr[2], dinv[2], del[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const size_t r = (size_t)bh * L + row0 + warp * 16 + g + 8 * h;
        mr[h] = mstat[r];
        dinv[h] = dinvstat[r];
        del[h] = delta[r];
    }
    const uint32_t* mrow = mask + ((size_t)bh * nblk + row0 / BS) * words;
    float acc[ND][4];
    zero(acc);
#pragma unroll 1
    for (int j = 0; j < nblk; ++j) {
        if (C::NST == 1) {
            __syncthreads();  // K_{j-1} and the dS in V's space no longer read
            stage_kv(j, 0);
            cp_commit();
        }
        cp_wait_all();
        __syncthreads();  // K_j, V_j visible to all; every warp has finished block j-1
        if (C::NST == 2 && j + 1 < nblk) {
            stage_kv(j + 1, (j + 1) & 1);
            cp_commit();
        }
        T* Ks = KV + (C::NST == 2 ? (j & 1) : 0) * 2 * BS * C::LD;
        T* Vs = Ks + BS * C::LD;
        float s[NS][4], gg[NS][4];
        zero(s);
        zero(gg);
        warp_mma_nk<NS, D>(s, Qs + warp * 16 * C::LD, C::LD, Ks, C::LD, lane);
        warp_mma_nk<NS, D>(gg, dOs + warp * 16 * C::LD, C::LD, Vs, C::LD, lane);
        row_grad<NS, BS>(s, gg, selected(mrow, j), order, gate, mr, dinv, del);
        __syncthreads();  // every warp has finished reading V_j: its space takes dS
        T* drow = Vs + warp * 16 * C::LDS;
#pragma unroll
        for (int nt = 0; nt < NS; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                st_pair(drow + (g + 8 * h) * C::LDS + nt * 8 + 2 * t, s[nt][2 * h], s[nt][2 * h + 1]);
        __syncwarp();
        warp_mma_kn<ND, BS>(acc, drow, C::LDS, Ks, C::LD, lane);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float* out = dq + hoff + (size_t)(row0 + warp * 16 + g + 8 * h) * D + 2 * t;
#pragma unroll
        for (int nt = 0; nt < ND; ++nt)
            *reinterpret_cast<float2*>(out + nt * 8) = make_float2(acc[nt][2 * h], acc[nt][2 * h + 1]);
    }
}

// ---------------------------------------------------------------------------
// dk, dv: key-major.  Per 32-row query chunk: S^T = K_j Q^T and G^T = V_j dO^T
// (warp w holds keys 16w .. 16w+15 of the block, the chunk's rows as columns),
// P^T and dS^T in registers, the block reductions of an unselected block over
// the 8 lanes of a column and then across the warps through shared memory,
// then dv += P^T dO and dk += dS^T Q.  The selection bit is the same for the
// whole chunk (its 32 rows lie in one query tile), so every thread takes the
// same branch and the barriers inside it are uniform.  The next chunk's Q, dO
// and row statistics load (cp.async) during this one.
// ---------------------------------------------------------------------------
template <typename T, int D, int BS>
__global__ void __launch_bounds__(BS * 2) bwd_dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v, const T* __restrict__ dO,
                                                          const uint32_t* __restrict__ mask, int L, int nblk,
                                                          int words, int order, int gate,
                                                          const float* __restrict__ mstat,
                                                          const float* __restrict__ dinvstat,
                                                          const float* __restrict__ delta, float* __restrict__ dk,
                                                          float* __restrict__ dv) {
    using C = Cfg<T, D, BS>;
    constexpr int NW = C::NW_KV, NTH = BS * 2, NC = kQC / 8, ND = D / 8;
    extern __shared__ __align__(16) unsigned char sm_bwd[];
    T* Ks = reinterpret_cast<T*>(sm_bwd);
    T* Vs = Ks + BS * C::LD;
    T* QD = Vs + BS * C::LD;                    // NST stages of (Q chunk, dO chunk)
    T* Ps = QD + 2 * C::NST * kQC * C::LD;
    T* dSs = Ps + BS * C::LDP;
    float* red = reinterpret_cast<float*>(sm_bwd + sizeof(T) * C::DKDV_T);  // [NW][kQC][4]
    float* stb = red + NW * kQC * 4;  // NST stages of [m | 1/D | delta] x kQC
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int j = blockIdx.x, bh = blockIdx.y;
    const size_t hoff = (size_t)bh * L * D;
    const int nchunk = L / kQC;
    auto stage_chunk = [&](int c, int st) {
        const int t0 = c * kQC;
        T* qs = QD + st * 2 * kQC * C::LD;
        cp_rows<T, D>(qs, C::LD, q + hoff + (size_t)t0 * D, kQC, tid, NTH);
        cp_rows<T, D>(qs + kQC * C::LD, C::LD, dO + hoff + (size_t)t0 * D, kQC, tid, NTH);
        float* sb_ = stb + st * 3 * kQC;
        const size_t r0 = (size_t)bh * L + t0;
        if (tid < 3 * kQC / 4) {  // 3 arrays x kQC floats in 16-byte pieces
            const int a = tid / (kQC / 4), p = (tid % (kQC / 4)) * 4;
            const float* src = (a == 0 ? mstat : a == 1 ? dinvstat : delta) + r0 + p;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(saddr(sb_ + a * kQC + p)), "l"(src)
                         : "memory");
        }
    };
    cp_rows<T, D>(Ks, C::LD, k + hoff + (size_t)j * BS * D, BS, tid, NTH);
    cp_rows<T, D>(Vs, C::LD, v + hoff + (size_t)j * BS * D, BS, tid, NTH);
    if (C::NST == 2) stage_chunk(0, 0);
    cp_commit();
    const float inv_b = 1.f / (float)BS, ln_b = logf((float)BS);
    const float c1 = order >= 1 ? 1.f : 0.f;
    float adk[ND][4], adv[ND][4];
    zero(adk);
    zero(adv);
#pragma unroll 1
    for (int c = 0; c < nchunk; ++c) {
        if (C::NST == 1) {
            __syncthreads();  // the previous chunk's tiles and statistics are no longer read
            stage_chunk(c, 0);
            cp_commit();
        }
        cp_wait_all();
        __syncthreads();  // chunk c visible to all; every warp has finished chunk c-1
        if (C::NST == 2 && c + 1 < nchunk) {
            stage_chunk(c + 1, (c + 1) & 1);
            cp_commit();
        }
        const int st_i = C::NST == 2 ? (c & 1) : 0;
        const T* Qs = QD + st_i * 2 * kQC * C::LD;
        const T* dOs = Qs + kQC * C::LD;
        const float* st = stb + st_i * 3 * kQC;
        float s[NC][4], gg[NC][4], p[NC][4];
        zero(s);
        zero(gg);
        warp_mma_nk2<NC, D>(s, Ks + warp * 16 * C::LD, Qs, gg, Vs + warp * 16 * C::LD, dOs, C::LD, C::LD, lane);
        const bool sel = selected(mask + ((size_t)bh * nblk + (c * kQC) / BS) * words, j);
        if (sel) {
#pragma unroll
            for (int nt = 0; nt < NC; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int cc = nt * 8 + 2 * t + e;
                    const float mc = st[cc], dic = st[kQC + cc], dc = st[2 * kQC + cc];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float pv = expf(s[nt][2 * h + e] - mc) * dic;
                        p[nt][2 * h + e] = pv;
                        s[nt][2 * h + e] = pv * (gg[nt][2 * h + e] - dc);
                    }
                }
        } else {
            // column sums of x over the block's keys: 16 per warp, then across the warps
#pragma unroll
            for (int nt = 0; nt < NC; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float part = col_sum(s[nt][e] + s[nt][2 + e]);
                    if (g == 0) red[(warp * kQC + nt * 8 + 2 * t + e) * 4] = part;
                }
            __syncthreads();
            float sb[NC][2];
#pragma unroll
            for (int nt = 0; nt < NC; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int cc = nt * 8 + 2 * t + e;
                    float tot = 0.f;
#pragma unroll
                    for (int w2 = 0; w2 < NW; ++w2) tot += red[(w2 * kQC + cc) * 4];
                    sb[nt][e] = tot * inv_b;
                    const float u0 = s[nt][e] - sb[nt][e], u1 = s[nt][2 + e] - sb[nt][e];
                    const float pv = col_sum(fmaf(u0, u0, u1 * u1));
                    const float pg = col_sum(gg[nt][e] + gg[nt][2 + e]);
                    const float pgu = col_sum(fmaf(gg[nt][e], u0, gg[nt][2 + e] * u1));
                    if (g == 0) {
                        float* rr = red + (warp * kQC + cc) * 4;
                        rr[1] = pv;
                        rr[2] = pg;
                        rr[3] = pgu;
                    }
                }
            __syncthreads();
#pragma unroll
            for (int nt = 0; nt < NC; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int cc = nt * 8 + 2 * t + e;
                    float sv = 0.f, sg = 0.f, sgu = 0.f;
#pragma unroll
                    for (int w2 = 0; w2 < NW; ++w2) {
                        const float* rr = red + (w2 * kQC + cc) * 4;
                        sv += rr[1];
                        sg += rr[2];
                        sgu += rr[3];
                    }
                    float w = 0.f, q2 = 0.f;
                    if (order == 2) {
                        w = sv * (0.5f * inv_b);
                        if (gate && w > ln_b) w = 0.f;
                        else q2 = inv_b;
                    }
                    const float a = expf(sb[nt][e] + w - st[cc]) * st[kQC + cc];
                    const float inner = sg + c1 * sgu - (float)BS * st[2 * kQC + cc];
                    const float gbar = sg * inv_b;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float u = s[nt][2 * h + e] - sb[nt][e];
                        p[nt][2 * h + e] = a * (1.f + c1 * u);
                        s[nt][2 * h + e] = a * ((inv_b + q2 * u) * inner + c1 * (gg[nt][2 * h + e] - gbar));
                    }
                }
        }
        T* prow = Ps + warp * 16 * C::LDP;
        T* drow = dSs + warp * 16 * C::LDP;
#pragma unroll
        for (int nt = 0; nt < NC; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int o2 = (g + 8 * h) * C::LDP + nt * 8 + 2 * t;
                st_pair(prow + o2, p[nt][2 * h], p[nt][2 * h + 1]);
                st_pair(drow + o2, s[nt][2 * h], s[nt][2 * h + 1]);
            }
        __syncwarp();
        warp_mma_kn<ND, kQC>(adv, prow, C::LDP, dOs, C::LD, lane);
        warp_mma_kn<ND, kQC>(adk, drow, C::LDP, Qs, C::LD, lane);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const size_t r = hoff + (size_t)(j * BS + warp * 16 + g + 8 * h) * D + 2 * t;
#pragma unroll
        for (int nt = 0; nt < ND; ++nt) {
            *reinterpret_cast<float2*>(dk + r + nt * 8) = make_float2(adk[nt][2 * h], adk[nt][2 * h + 1]);
            *reinterpret_cast<float2*>(dv + r + nt * 8) = make_float2(adv[nt][2 * h], adv[nt][2 * h + 1]);
        }
    }
}

}  // namespace bwd
}  // namespace pisa
