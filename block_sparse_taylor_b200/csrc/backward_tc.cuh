// Backward pass of the piecewise sparse attention on tcgen05 tensor cores
// (bf16 inputs): the gradients dq, dk, dv of sum_t dO_t . o_t, with the block
// selection held fixed (the same derivative as backward.cuh; the pages define
// only the forward: PISA paper section 3.2 "Formulation"; "Sparse Linear
// Attention" blog, the sparse-linear and PWT sections).
//
// Per query row t (x_n = q_t.k_n, G_n = dO_t.v_n, delta = dO_t.o_t, lse_t = ln D_t
// the forward's log-denominator):
//   selected key n           P_n = e^{x_n - lse_t},       dS_n = P_n (G_n - delta)
//   key n of unselected j    sb = mean_n x_n, u_n = x_n - sb, l = sb + w
//                            (w = [order 2] sum u^2 / 2B, zeroed by the gate),
//                            a = e^{l - lse_t},  P_n = a (1 + c1 u_n),
//                            inner = sum_n G_n (1 + c1 u_n) - B delta,
//                            dS_n = a (dl_n inner + c1 (G_n - mean G)),
//                            dl_n = 1/B (+ u_n / B for order 2 with the gate open)
//   dq_t = sum_n dS_tn k_n,   dk_n = sum_t dS_tn q_t,   dv_n = sum_t P_tn dO_t
// (c1 = 1 for order >= 1, 0 for order 0).
//
// bwd_dq_tc_kernel (query-major): one 128-row M tile of one (batch, head) per
// CTA, visiting every key tile of 128 keys.  Every reduction over a block
// (sb, sum G, sum G u, the spread behind w) runs over the block's keys of one
// query row, which are TMEM columns of one lane.
//   warp 0      TMA producer: Q and dO once; K tiles through three stages, V
//               tiles through two (V is free once G = dO V^T has completed)
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2-9   softmax: warp w takes lane quarter w % 4 and key half (w - 2) / 4
//               of each tile, 64 keys: it loads its S and G columns into
//               registers with one wait, releases G, forms the block sums in
//               one shifted pass (at B = 128 the two halves of a block add their
//               sums through four spare TMEM columns), and writes dS in bf16 over
//               the first 32 of its S columns
// TMEM: S_0 | S_1 | G | dQ.  S = Q K^T alternates between two buffers; dQ +=
// dS K runs from TMEM (K as the MN-major B operand).  MMA order per tile j:
// G_{j+1} as soon as the softmax holds G_j in registers, then dQ_j and S_{j+2}
// once dS_j is written, so the next G product runs beside the softmax.
#pragma once

#include <cudaTypedefs.h>

#include <string>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace pisa {
namespace bwdtc {

constexpr int kThreads = 320;  // producer, MMA issuer, eight softmax warps (two per lane quarter)

template <int D>
struct DqCfg {
    static constexpr int NK = 128;
    static constexpr int NBOX = D / 64;
    static constexpr uint32_t BOX_BYTES = 128 * 128;  // 128 rows x 128 bytes
    static constexpr uint32_t TILE_BYTES = NBOX * BOX_BYTES;
    static constexpr int NSK = 3, NSV = 2;             // K and V stages
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t DO_OFF = Q_OFF + TILE_BYTES;
    static constexpr uint32_t K_OFF = DO_OFF + TILE_BYTES;
    static constexpr uint32_t V_OFF = K_OFF + NSK * TILE_BYTES;
    static constexpr uint32_t BAR_OFF = V_OFF + NSV * TILE_BYTES;
    // QFULL; KFULL, KEMPTY per K stage; VFULL, VEMPTY per V stage; SFULL, DSREADY per
    // S buffer; GFULL, GFREE; DQFULL; DONE; PAIR per lane quarter (B = 128 block sums)
    static constexpr uint32_t NBAR = 1 + 2 * NSK + 2 * NSV + 4 + 2 + 1 + 1 + 4;
    static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
    static constexpr uint32_t G_COL = 256, DQ_COL = 384;
    static constexpr uint32_t TMEM_COLS = 512;
};

// delta_t = dO_t . o_t (one warp per row, fp32 accumulation)
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const bf16* __restrict__ o, const bf16* __restrict__ dO,
                                                        long rows, float* __restrict__ delta) {
    const long row = (long)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= rows) return;
    const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(o + row * D);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(dO + row * D);
    float s = 0.f;
#pragma unroll
    for (int c = lane; c < D / 2; c += 32) {
        const float2 x = __bfloat1622float2(a[c]), y = __bfloat1622float2(b[c]);
        s = fmaf(x.x, y.x, fmaf(x.y, y.y, s));
    }
    s = warp_sum(s);
    if (lane == 0) delta[row] = s;
}

// lse_t = m_t + ln D_t from the row statistics kernel's m_t and 1/D_t
__global__ void bwd_lse_kernel(const float* __restrict__ m, const float* __restrict__ dinv, long n,
                               float* __restrict__ lse) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
        lse[i] = m[i] - logf(dinv[i]);
}

// Block sums of one query row over the 64 keys of a half tile that this thread holds
// (S and G as raw fp32 bits, two 32-key chunks each), in one pass shifted by x0, the
// block's first logit (the shift keeps the sums of (x - x0) free of cancellation when the
// block's logits share a large offset):
//   s1 = sum (x - x0), s2 = sum (x - x0)^2, sg = sum G, sgd = sum G (x - x0)
// so that sb = x0 + s1/B, sum (x - sb)^2 = s2 - s1^2/B, sum G (x - sb) = sgd - (s1/B) sg.
// Packed fp32 pairs: the even and the odd keys accumulate separately.
struct HalfSums {
    float s1, s2, sg, sgd;
};

__device__ __forceinline__ HalfSums half_sums(const uint32_t (&xa)[32], const uint32_t (&xb)[32],
                                              const uint32_t (&ga)[32], const uint32_t (&gb)[32], float x0) {
    const uint64_t nx0 = tc::f2_make(-x0, -x0);
    uint64_t a1 = 0ull, a2 = 0ull, ag = 0ull, agd = 0ull;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const uint32_t* xs = e < 16 ? xa : xb;
        const uint32_t* gs = e < 16 ? ga : gb;
        const int o = 2 * (e & 15);
        const uint64_t x2 = tc::f2_make(__uint_as_float(xs[o]), __uint_as_float(xs[o + 1]));
        const uint64_t g2 = tc::f2_make(__uint_as_float(gs[o]), __uint_as_float(gs[o + 1]));
        const uint64_t dx = tc::f2_add(x2, nx0);
        a1 = tc::f2_add(a1, dx);
        a2 = tc::f2_fma(dx, dx, a2);
        ag = tc::f2_add(ag, g2);
        agd = tc::f2_fma(g2, dx, agd);
    }
    const float2 s1 = tc::f2_split(a1), s2 = tc::f2_split(a2), sg = tc::f2_split(ag), sgd = tc::f2_split(agd);
    return HalfSums{s1.x + s1.y, s2.x + s2.y, sg.x + sg.y, sgd.x + sgd.y};
}

// dS of 32 keys (one chunk of a half tile), packed as bf16 pairs (keys 2e, 2e + 1 in word
// e).  Selected block: P = 2^{x log2 e - lse2}, dS = P (G - delta); unselected block:
// u = x - sb, dS = A G + X u + Cc.  The test of `sel` stays outside the loops (it is the
// same for the 32 rows of a warp), so that only selected rows pay for the exponentials.
// A row past the sequence end comes in with lse2 = +inf and delta = 0: every term is 0.
__device__ __forceinline__ void chunk_ds(const uint32_t (&xs)[32], const uint32_t (&gs)[32], bool sel, float lse2,
                                         float del, float sb, float A, float X, float Cc, uint32_t (&dd)[16]) {
    constexpr float LOG2E = 1.4426950408889634f;
    if (sel) {
        const uint64_t ndel = tc::f2_make(-del, -del);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint64_t g2 = tc::f2_make(__uint_as_float(gs[2 * e]), __uint_as_float(gs[2 * e + 1]));
            const uint64_t p2 = tc::f2_make(tc::ex2(fmaf(__uint_as_float(xs[2 * e]), LOG2E, -lse2)),
                                            tc::ex2(fmaf(__uint_as_float(xs[2 * e + 1]), LOG2E, -lse2)));
            const float2 d = tc::f2_split(tc::f2_mul(p2, tc::f2_add(g2, ndel)));
            dd[e] = tc::pack_bf16x2(d.x, d.y);
        }
    } else {
        const uint64_t nsb = tc::f2_make(-sb, -sb);
        const uint64_t A2 = tc::f2_make(A, A), X2 = tc::f2_make(X, X), C2 = tc::f2_make(Cc, Cc);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint64_t g2 = tc::f2_make(__uint_as_float(gs[2 * e]), __uint_as_float(gs[2 * e + 1]));
            const uint64_t u2 = tc::f2_add(tc::f2_make(__uint_as_float(xs[2 * e]), __uint_as_float(xs[2 * e + 1])), nsb);
            const float2 d = tc::f2_split(tc::f2_fma(A2, g2, tc::f2_fma(X2, u2, C2)));
            dd[e] = tc::pack_bf16x2(d.x, d.y);
        }
    }
}

// Per-block coefficients from the sums: sb (mean logit), a = e^{l - lse} (l = sb + w),
// and dS_n = A G_n + X u_n + Cc, P_n = a + Pu u_n for an unselected block (u_n = x_n - sb);
// `inner` = sum_n G_n (1 + c1 u_n) - B delta, so that dL/dl = a inner.  ORDER 3 is the first
// order with PWT's pooled w (wp, the tile's gated value for this block): it does not depend
// on the row's logits, so dl_n = 1/B.
template <int BS, int ORDER>
__device__ __forceinline__ void block_coefs(float x0, float s1, float s2, float sg, float sgd, float lse2, float del,
                                            int gate, float ln_b, float wp, float& sb, float& a, float& A, float& X,
                                            float& Cc, float& Pu, float& inner) {
    constexpr float LOG2E = 1.4426950408889634f;
    constexpr float INV_B = 1.0f / (float)BS;
    constexpr float C1 = ORDER >= 1 ? 1.f : 0.f;
    const float md = s1 * INV_B;
    sb = x0 + md;
    float w = 0.f, q2 = 0.f;
    if (ORDER == 2) {
        // w = (1/2B) sum (x - sb)^2 and the forward's gate decision held fixed: dl_n carries
        // u_n / B only where w was kept
        w = 0.5f * fmaxf(fmaf(-md, s1, s2), 0.f) * INV_B;
        if (gate && w > ln_b) {
            w = 0.f;
        } else {
            q2 = INV_B;
        }
    } else if (ORDER == 3) {
        w = wp;
    }
    a = tc::ex2((sb + w) * LOG2E - lse2);
    const float sgu = fmaf(-md, sg, sgd);  // sum G (x - sb)
    inner = sg + C1 * sgu - (float)BS * del;
    // dS_n = a (dl_n inner + c1 (G_n - mean G)),  dl_n = 1/B (+ q2 u_n)
    A = a * C1;
    X = a * q2 * inner;
    Cc = a * (INV_B * inner - C1 * sg * INV_B);
    Pu = a * C1;
}

template <int D, int BS, int ORDER>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const uint32_t* __restrict__ mask, const float* __restrict__ lse,
                     const float* __restrict__ delta, float* __restrict__ dq, int L, int nblk, int words, int gate,
                     unsigned* status, const float* __restrict__ wmat, float* __restrict__ wpart) {
    // ORDER 3 (first order + PWT's pooled w): wmat [BH, nblk, nblk] the gated w of each (query
    // tile, block); wpart [BH, L / 32, nblk] receives, per 32 query rows and block, the sum of
    // dL/dl over those rows (0 for selected blocks and blocks whose w is 0), the pooled w's
    // gradient before it reaches q and k
    using C = DqCfg<D>;
    constexpr float LOG2E = 1.4426950408889634f;
    constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, false);  // S = Q K^T, G = dO V^T
    constexpr uint32_t IDESC_Q = tc::idesc_bf16(128, D, true);     // dQ += dS K, K MN-major

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_addr(smem);
    auto bar = [&](int i) { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
    const int B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 1 + C::NSK, B_VFULL = 1 + 2 * C::NSK,
              B_VEMPTY = B_VFULL + C::NSV, B_SFULL = B_VEMPTY + C::NSV, B_DSREADY = B_SFULL + 2,
              B_GFULL = B_DSREADY + 2, B_GFREE = B_GFULL + 1, B_DQFULL = B_GFREE + 1, B_DONE = B_DQFULL + 1,
              B_PAIR = B_DONE + 1;
    uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + C::NBAR * 8);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = blockIdx.y;
    const int q0 = blockIdx.x * 128;
    const int NT = L / C::NK;
    bool aborted = false;

    if (threadIdx.x == 0) {
        tc::mbar_init(bar(B_QFULL), 1);
        for (int s = 0; s < C::NSK; ++s) {
            tc::mbar_init(bar(B_KFULL + s), 1);
            tc::mbar_init(bar(B_KEMPTY + s), 1);
        }
        for (int s = 0; s < C::NSV; ++s) {
            tc::mbar_init(bar(B_VFULL + s), 1);
            tc::mbar_init(bar(B_VEMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(bar(B_SFULL + b), 1);
            tc::mbar_init(bar(B_DSREADY + b), 256);
        }
        tc::mbar_init(bar(B_GFULL), 1);
        tc::mbar_init(bar(B_GFREE), 256);
        tc::mbar_init(bar(B_DQFULL), 1);
        tc::mbar_init(bar(B_DONE), 1);
        for (int qq = 0; qq < 4; ++qq) tc::mbar_init(bar(B_PAIR + qq), 64);
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tc::tma_prefetch(&tm_q);
            tc::tma_prefetch(&tm_k);
            tc::tma_prefetch(&tm_v);
            tc::tma_prefetch(&tm_do);
            const int row0 = bh * L + q0;
            tc::mbar_expect_tx(bar(B_QFULL), 2 * C::TILE_BYTES);
            for (int b = 0; b < C::NBOX; ++b) {
                tc::tma_load_2d(sbase + C::Q_OFF + b * C::BOX_BYTES, &tm_q, bar(B_QFULL), b * 64, row0);
                tc::tma_load_2d(sbase + C::DO_OFF + b * C::BOX_BYTES, &tm_do, bar(B_QFULL), b * 64, row0);
            }
            int lastK = -1, lastV = -1;
            for (int j = 0; j < NT; ++j) {
                const int sk = j % C::NSK, uk = j / C::NSK, sv = j % C::NSV, uv = j / C::NSV;
                if (uk > 0 && !tc::mbar_wait(bar(B_KEMPTY + sk), (uk - 1) & 1, aborted, status, kWaitLimitCycles))
                    break;
                tc::mbar_expect_tx(bar(B_KFULL + sk), C::TILE_BYTES);
                for (int b = 0; b < C::NBOX; ++b)
                    tc::tma_load_2d(sbase + C::K_OFF + sk * C::TILE_BYTES + b * C::BOX_BYTES, &tm_k, bar(B_KFULL + sk),
                                    b * 64, bh * L + j * C::NK);
                lastK = j;
                if (uv > 0 && !tc::mbar_wait(bar(B_VEMPTY + sv), (uv - 1) & 1, aborted, status, kWaitLimitCycles))
                    break;
                tc::mbar_expect_tx(bar(B_VFULL + sv), C::TILE_BYTES);
                for (int b = 0; b < C::NBOX; ++b)
                    tc::tma_load_2d(sbase + C::V_OFF + sv * C::TILE_BYTES + b * C::BOX_BYTES, &tm_v, bar(B_VFULL + sv),
                                    b * 64, bh * L + j * C::NK);
                lastV = j;
            }
            if (aborted) {
                // let every copy already issued land before the CTA exits
                bool a2 = false;
                tc::mbar_wait(bar(B_QFULL), 0, a2, status, kWaitLimitCycles);
                for (int j = (lastK - C::NSK + 1 > 0 ? lastK - C::NSK + 1 : 0); j <= lastK; ++j) {
                    a2 = false;
                    tc::mbar_wait(bar(B_KFULL + j % C::NSK), (j / C::NSK) & 1, a2, status, kWaitLimitCycles);
                }
                for (int j = (lastV - C::NSV + 1 > 0 ? lastV - C::NSV + 1 : 0); j <= lastV; ++j) {
                    a2 = false;
                    tc::mbar_wait(bar(B_VFULL + j % C::NSV), (j / C::NSV) & 1, a2, status, kWaitLimitCycles);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint64_t qdesc = tc::sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
            const uint64_t dodesc = tc::sdesc_sw128(sbase + C::DO_OFF, 16, 1024);
            const uint64_t kdesc0 = tc::sdesc_sw128(sbase + C::K_OFF, 16, 1024);
            const uint64_t kmn0 = tc::sdesc_sw128(sbase + C::K_OFF, C::BOX_BYTES, 1024);  // K as MN-major B
            const uint64_t vdesc0 = tc::sdesc_sw128(sbase + C::V_OFF, 16, 1024);
            constexpr uint64_t kTileStep = C::TILE_BYTES >> 4;
            // D[dcol] = A (Q or dO) x B^T (K or V tile), K-dim = d
            auto issue_kd = [&](uint32_t dcol, uint64_t adesc, uint64_t bdesc) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
                    tc::mma_ss(tmem + dcol, adesc + off, bdesc + off, IDESC_S, kk > 0);
                }
            };
            // dQ += dS (TMEM, buffer b) x K_j (MN-major), K-dim = 128 keys.  dS of keys
            // 64h .. 64h + 63 sits packed in columns 64h .. 64h + 31 of the buffer.
            auto issue_dq = [&](int b, int sk, bool first) {
#pragma unroll
                for (int kk = 0; kk < C::NK / 16; ++kk)
                    tc::mma_ts(tmem + C::DQ_COL, tmem + (uint32_t)(b * 128 + kk * 8 + (kk >= 4 ? 32 : 0)),
                               kmn0 + sk * kTileStep + (uint64_t)((kk * 16 * 128) >> 4), IDESC_Q,
                               (first && kk == 0) ? 0u : 1u);
            };
            bool ok = tc::mbar_wait(bar(B_QFULL), 0, aborted, status, kWaitLimitCycles);
            // prologue: S_0, G_0, S_1
            ok = ok && tc::mbar_wait(bar(B_KFULL + 0), 0, aborted, status, kWaitLimitCycles);
            if (ok) {
                issue_kd(0, qdesc, kdesc0);
                tc::mma_commit(bar(B_SFULL + 0));
            }
            ok = ok && tc::mbar_wait(bar(B_VFULL + 0), 0, aborted, status, kWaitLimitCycles);
            if (ok) {
                issue_kd(C::G_COL, dodesc, vdesc0);
                tc::mma_commit(bar(B_GFULL));
                tc::mma_commit(bar(B_VEMPTY + 0));
            }
            if (ok && NT > 1) {
                ok = tc::mbar_wait(bar(B_KFULL + 1), 0, aborted, status, kWaitLimitCycles);
                if (ok) {
                    issue_kd(128, qdesc, kdesc0 + 1 * kTileStep);
                    tc::mma_commit(bar(B_SFULL + 1));
                }
            }
            for (int j = 0; ok && j < NT; ++j) {
                const int b = j & 1;
                // the softmax has read G_j (and S_j) into registers: G_{j+1} may overwrite it
                if (!tc::mbar_wait(bar(B_GFREE), j & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                if (j + 1 < NT) {
                    const int sv = (j + 1) % C::NSV, uv = (j + 1) / C::NSV;
                    if (!tc::mbar_wait(bar(B_VFULL + sv), uv & 1, aborted, status, kWaitLimitCycles)) break;
                    issue_kd(C::G_COL, dodesc, vdesc0 + sv * kTileStep);
                    tc::mma_commit(bar(B_GFULL));
                    tc::mma_commit(bar(B_VEMPTY + sv));
                }
                // the softmax of tile j has written dS_j
                if (!tc::mbar_wait(bar(B_DSREADY + b), (j >> 1) & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                issue_dq(b, j % C::NSK, j == 0);
                tc::mma_commit(bar(B_KEMPTY + j % C::NSK));
                if (j + 2 < NT) {
                    const int sk = (j + 2) % C::NSK, uk = (j + 2) / C::NSK;
                    if (!tc::mbar_wait(bar(B_KFULL + sk), uk & 1, aborted, status, kWaitLimitCycles)) break;
                    issue_kd((uint32_t)(b * 128), qdesc, kdesc0 + sk * kTileStep);
                    tc::mma_commit(bar(B_SFULL + b));
                }
            }
            if (!aborted) tc::mma_commit(bar(B_DQFULL));
            // every MMA issued by this thread has completed before TMEM is freed
            tc::mma_commit(bar(B_DONE));
            bool a2 = false;
            tc::mbar_wait(bar(B_DONE), 0, a2, status, kWaitLimitCycles);
        }
    } else {
        // ------------------------------------------------------------- softmax
        // Warp w takes lane quarter w % 4 (32 query rows) and key half (w - 2) / 4 of every
        // tile: 64 keys, one block at B = 64, half of one at B = 128 (whose sums the two warps
        // of a quarter exchange).
        const int quarter = warp % 4;
        const int half = (warp - 2) / 4;
        const int r = quarter * 32 + lane;      // row inside the M tile = TMEM lane
        const int qrow = q0 + r;
        const bool valid = qrow < L;
        const int qt = (valid ? qrow : L - 1) / BS;  // query tile (selection row)
        const uint32_t* mrow = mask + ((size_t)bh * nblk + qt) * words;
        // log2 units; +inf past the sequence end, where it makes every coefficient 0
        const float lse2 = valid ? __ldg(lse + (size_t)bh * L + qrow) * LOG2E : __int_as_float(0x7f800000);
        const float del = valid ? __ldg(delta + (size_t)bh * L + qrow) : 0.f;
        const float ln_b = logf((float)BS);
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t g_addr = lane_base + C::G_COL + 64 * half;
        for (int j = 0; j < NT; ++j) {
            const int b = j & 1;
            if (!tc::mbar_wait_warp(bar(B_SFULL + b), (j >> 1) & 1, aborted, status, kWaitLimitCycles)) break;
            if (!tc::mbar_wait_warp(bar(B_GFULL), j & 1, aborted, status, kWaitLimitCycles)) break;
            tc::fence_after_sync();
            const uint32_t s_tile = lane_base + (uint32_t)(b * 128);
            const uint32_t s_addr = s_tile + 64 * half;
            uint32_t xa[32], xb[32], ga[32], gb[32];
            tc::tmem_ld32(s_addr, xa);
            tc::tmem_ld32(s_addr + 32, xb);
            tc::tmem_ld32(g_addr, ga);
            tc::tmem_ld32(g_addr + 32, gb);
            uint32_t x0raw = 0u;
            if (BS == 128 && half == 1) x0raw = tc::tmem_ld1(s_tile);  // the block's first logit
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_GFREE));
            const int jb = (j * C::NK + 64 * half) / BS;  // this half's block
            const bool sel = (__ldg(mrow + (jb >> 5)) >> (jb & 31)) & 1u;
            const float x0 = (BS == 128 && half == 1) ? __uint_as_float(x0raw) : __uint_as_float(xa[0]);
            HalfSums hs = half_sums(xa, xb, ga, gb, x0);
            if (BS == 128) {
                // the other half's sums, through four TMEM columns of this buffer that hold
                // S of keys this warp has already read (the dS columns are the first 32)
                uint32_t mine[4] = {__float_as_uint(hs.s1), __float_as_uint(hs.s2), __float_as_uint(hs.sg),
                                    __float_as_uint(hs.sgd)};
                tc::tmem_st4(s_addr + 32, mine);
                tc::tmem_wait_st();
                tc::fence_before_sync();
                tc::mbar_arrive(bar(B_PAIR + quarter));
                if (!tc::mbar_wait_warp(bar(B_PAIR + quarter), j & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                uint32_t other[4];
                tc::tmem_ld4(s_tile + 64 * (1 - half) + 32, other);
                tc::tmem_wait_ld();
                hs.s1 += __uint_as_float(other[0]);
                hs.s2 += __uint_as_float(other[1]);
                hs.sg += __uint_as_float(other[2]);
                hs.sgd += __uint_as_float(other[3]);
            }
            float sb, a, A, X, Cc, Pu, inner;
            const float wp = (ORDER == 3) ? __ldg(wmat + ((size_t)bh * nblk + qt) * nblk + jb) : 0.f;
            block_coefs<BS, ORDER>(x0, hs.s1, hs.s2, hs.sg, hs.sgd, lse2, del, gate, ln_b, wp, sb, a, A, X, Cc, Pu,
                                   inner);
            if (ORDER == 3) {
                float gw = (!sel && valid && wp > 0.f) ? a * inner : 0.f;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) gw += __shfl_xor_sync(0xffffffffu, gw, o);
                if (lane == 0 && (BS == 64 || half == 0))
                    wpart[((size_t)bh * (L / 32) + (q0 / 32 + quarter)) * nblk + jb] = gw;
            }
            // dS (bf16) over the first 32 columns of this half: keys 2e and 2e + 1 in column e
            {
                uint32_t dd[16];
                chunk_ds(xa, ga, sel, lse2, del, sb, A, X, Cc, dd);
                tc::tmem_st16(s_addr, dd);
                chunk_ds(xb, gb, sel, lse2, del, sb, A, X, Cc, dd);
                tc::tmem_st16(s_addr + 16, dd);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_DSREADY + b));
        }
        // epilogue: this warp's column half of the dq row (fp32) to global
        if (tc::mbar_wait_warp(bar(B_DQFULL), 0, aborted, status, kWaitLimitCycles)) {
            tc::fence_after_sync();
            float* drow = dq + ((size_t)bh * L + (valid ? qrow : 0)) * D + half * (D / 2);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t raw[32];
                tc::tmem_ld32(lane_base + C::DQ_COL + half * (D / 2) + c * 32, raw);
                tc::tmem_wait_ld();
                if (valid) {
                    float4* dst = reinterpret_cast<float4*>(drow + c * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(__uint_as_float(raw[4 * e]), __uint_as_float(raw[4 * e + 1]),
                                             __uint_as_float(raw[4 * e + 2]), __uint_as_float(raw[4 * e + 3]));
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// bwd_dkdv_tc_kernel (key-major): one tile of 128 keys of one (batch, head) per
// CTA, visiting every query tile of 128 rows.  S = Q K^T and G = dO V^T are
// computed with the queries as TMEM lanes (the same orientation as the dq
// kernel), so every reduction over a block's keys stays inside one thread.  The
// softmax threads write P and dS (bf16) as rows of query t into shared memory
// in the 128-byte-swizzled layout of a TMA tile; read with the keys as the
// contiguous dimension, that is the MN-major A operand of
//   dV += P^T dO,   dK += dS^T Q     (M = the 128 keys, N = d, K-dim = queries)
// with dO and Q as MN-major B operands.  TMEM: S | G | dV | dK.
//   warp 0      TMA producer: K and V once; Q and dO tiles through their stages
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2-9   softmax: warp w takes lane quarter w % 4 (query rows, then key
//               rows in the epilogue of dK and dV) and key half (w - 2) / 4.
// Per query tile the softmax works in two passes: from S alone it forms the
// block sums of the logits, the coefficients that P needs and P itself, writes P
// (the dV product can start) and only then reads G for the sums of G, the rest
// of the coefficients and dS.  S and G are released as soon as they are in
// registers, so S of the next tile, and G where dO has a second stage, run beside
// the softmax.  MMA issue order per tile i:
//   S_{i+1} (two Q stages), dV_i, G_{i+1} (two dO stages), dK_i,
//   S_{i+1} (one Q stage: Q_{i+1} lands once dK_i has read Q_i),
//   G_{i+1} (one dO stage: dO_{i+1} lands once dV_i has read dO_i).
// Shared memory at d = 128 holds K, V, P, dS and three tiles of Q and dO: two Q
// stages at B = 64, one (and the B = 128 exchange buffer) at B = 128.
// ---------------------------------------------------------------------------
template <int D, int BS>
struct DkvCfg {
    static constexpr int NQ = 128;                     // query rows per tile
    static constexpr int NBOX = D / 64;
    static constexpr uint32_t BOX_BYTES = 128 * 128;
    static constexpr uint32_t TILE_BYTES = NBOX * BOX_BYTES;  // 128 rows x d bf16
    static constexpr uint32_t PT_BYTES = 2 * BOX_BYTES;       // 128 queries x 128 keys bf16
    static constexpr int NSQ = (D == 128 && BS == 128) ? 1 : 2;
    static constexpr int NSO = (D == 128) ? 1 : 2;
    static constexpr uint32_t K_OFF = 0;
    static constexpr uint32_t V_OFF = K_OFF + TILE_BYTES;
    static constexpr uint32_t Q_OFF = V_OFF + TILE_BYTES;
    static constexpr uint32_t DO_OFF = Q_OFF + NSQ * TILE_BYTES;
    static constexpr uint32_t P_OFF = DO_OFF + NSO * TILE_BYTES;
    static constexpr uint32_t DS_OFF = P_OFF + PT_BYTES;
    // B = 128: the two halves of a block add their sums through shared memory, twice a
    // tile (logit sums, then G sums): fp32 [exchange][key half][128 rows][2]
    static constexpr uint32_t XCH_OFF = DS_OFF + PT_BYTES;
    static constexpr uint32_t XCH_BYTES = (BS == 128) ? 2 * 2 * 128 * 2 * 4 : 0;
    static constexpr uint32_t BAR_OFF = XCH_OFF + XCH_BYTES;
    // KVFULL; QFULL, QEMPTY per Q stage; DOFULL, DOEMPTY per dO stage; SFULL, GFULL, SFREE,
    // GFREE, PREADY, DSREADY, PFREE, DSFREE, DKVFULL, DONE; PAIR per lane quarter
    static constexpr uint32_t NBAR = 1 + 2 * NSQ + 2 * NSO + 10 + 4;
    static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
    static constexpr uint32_t G_COL = 128, DV_COL = 256, DK_COL = 256 + D;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(SMEM <= 232448, "shared memory over the per-CTA limit");
};

// 16 bytes (8 bf16) at chunk c of row t of a 128-byte-swizzled tile (64 columns per box)
__device__ __forceinline__ void st_swz16(uint8_t* tile, int t, int col8, uint4 v) {
    const int box = col8 >> 3, c = col8 & 7;
    *reinterpret_cast<uint4*>(tile + box * (128 * 128) + t * 128 + ((c ^ (t & 7)) << 4)) = v;
}

// Sums of (x - x0) and (x - x0)^2 over the 64 logits of a half tile (packed pairs).
__device__ __forceinline__ float2 half_logit_sums(const uint32_t (&xa)[32], const uint32_t (&xb)[32], float x0) {
    const uint64_t nx0 = tc::f2_make(-x0, -x0);
    uint64_t a1 = 0ull, a2 = 0ull;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const uint32_t* xs = e < 16 ? xa : xb;
        const int o = 2 * (e & 15);
        const uint64_t dx = tc::f2_add(tc::f2_make(__uint_as_float(xs[o]), __uint_as_float(xs[o + 1])), nx0);
        a1 = tc::f2_add(a1, dx);
        a2 = tc::f2_fma(dx, dx, a2);
    }
    const float2 s1 = tc::f2_split(a1), s2 = tc::f2_split(a2);
    return make_float2(s1.x + s1.y, s2.x + s2.y);
}

// Sums of G and G (x - x0) over the half tile.
__device__ __forceinline__ float2 half_g_sums(const uint32_t (&xa)[32], const uint32_t (&xb)[32],
                                              const uint32_t (&ga)[32], const uint32_t (&gb)[32], float x0) {
    const uint64_t nx0 = tc::f2_make(-x0, -x0);
    uint64_t ag = 0ull, agd = 0ull;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const uint32_t* xs = e < 16 ? xa : xb;
        const uint32_t* gs = e < 16 ? ga : gb;
        const int o = 2 * (e & 15);
        const uint64_t dx = tc::f2_add(tc::f2_make(__uint_as_float(xs[o]), __uint_as_float(xs[o + 1])), nx0);
        const uint64_t g2 = tc::f2_make(__uint_as_float(gs[o]), __uint_as_float(gs[o + 1]));
        ag = tc::f2_add(ag, g2);
        agd = tc::f2_fma(g2, dx, agd);
    }
    const float2 sg = tc::f2_split(ag), sgd = tc::f2_split(agd);
    return make_float2(sg.x + sg.y, sgd.x + sgd.y);
}

// P of 32 keys from the logits alone (selected: 2^{x log2 e - lse2}; unselected: a + Pu u),
// with the same warp-uniform branch and the same zero rows past the sequence end as chunk_ds.
__device__ __forceinline__ void chunk_p(const uint32_t (&xs)[32], bool sel, float lse2, float sb, float a, float Pu,
                                        uint32_t (&pp)[16]) {
    constexpr float LOG2E = 1.4426950408889634f;
    if (sel) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
            pp[e] = tc::pack_bf16x2(tc::ex2(fmaf(__uint_as_float(xs[2 * e]), LOG2E, -lse2)),
                                    tc::ex2(fmaf(__uint_as_float(xs[2 * e + 1]), LOG2E, -lse2)));
    } else {
        const uint64_t nsb = tc::f2_make(-sb, -sb), a2 = tc::f2_make(a, a), P2 = tc::f2_make(Pu, Pu);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint64_t u2 = tc::f2_add(tc::f2_make(__uint_as_float(xs[2 * e]), __uint_as_float(xs[2 * e + 1])), nsb);
            const float2 p = tc::f2_split(tc::f2_fma(P2, u2, a2));
            pp[e] = tc::pack_bf16x2(p.x, p.y);
        }
    }
}

template <int D, int BS, int ORDER>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const uint32_t* __restrict__ mask, const float* __restrict__ lse,
                       const float* __restrict__ delta, float* __restrict__ dk, float* __restrict__ dv, int L,
                       int nblk, int words, int gate, unsigned* status, const float* __restrict__ wmat) {
    using C = DkvCfg<D, BS>;
    constexpr float LOG2E = 1.4426950408889634f;
    constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, false);
    // M = 128 keys, N = d, A (P or dS) and B (dO or Q) both MN-major
    constexpr uint32_t IDESC_KV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                  ((uint32_t)(D >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    constexpr bool kEarlyS = C::NSQ >= 2, kEarlyG = C::NSO >= 2;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_addr(smem);
    auto bar = [&](int i) { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
    const int B_KVFULL = 0, B_QFULL = 1, B_QEMPTY = B_QFULL + C::NSQ, B_DOFULL = B_QEMPTY + C::NSQ,
              B_DOEMPTY = B_DOFULL + C::NSO, B_SFULL = B_DOEMPTY + C::NSO, B_GFULL = B_SFULL + 1,
              B_SFREE = B_GFULL + 1, B_GFREE = B_SFREE + 1, B_PREADY = B_GFREE + 1, B_DSREADY = B_PREADY + 1,
              B_PFREE = B_DSREADY + 1, B_DSFREE = B_PFREE + 1, B_DKVFULL = B_DSFREE + 1, B_DONE = B_DKVFULL + 1,
              B_PAIR = B_DONE + 1;
    uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + C::NBAR * 8);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = blockIdx.y;
    const int k0 = blockIdx.x * 128;  // first key of this tile
    const int NQT = (L + C::NQ - 1) / C::NQ;
    bool aborted = false;

    if (threadIdx.x == 0) {
        tc::mbar_init(bar(B_KVFULL), 1);
        for (int s = 0; s < C::NSQ; ++s) {
            tc::mbar_init(bar(B_QFULL + s), 1);
            tc::mbar_init(bar(B_QEMPTY + s), 1);
        }
        for (int s = 0; s < C::NSO; ++s) {
            tc::mbar_init(bar(B_DOFULL + s), 1);
            tc::mbar_init(bar(B_DOEMPTY + s), 1);
        }
        tc::mbar_init(bar(B_SFULL), 1);
        tc::mbar_init(bar(B_GFULL), 1);
        tc::mbar_init(bar(B_SFREE), 256);
        tc::mbar_init(bar(B_GFREE), 256);
        tc::mbar_init(bar(B_PREADY), 256);
        tc::mbar_init(bar(B_DSREADY), 256);
        tc::mbar_init(bar(B_PFREE), 1);
        tc::mbar_init(bar(B_DSFREE), 1);
        tc::mbar_init(bar(B_DKVFULL), 1);
        tc::mbar_init(bar(B_DONE), 1);
        for (int qq = 0; qq < 4; ++qq) tc::mbar_init(bar(B_PAIR + qq), 64);
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tc::tma_prefetch(&tm_q);
            tc::tma_prefetch(&tm_k);
            tc::tma_prefetch(&tm_v);
            tc::tma_prefetch(&tm_do);
            tc::mbar_expect_tx(bar(B_KVFULL), 2 * C::TILE_BYTES);
            for (int b = 0; b < C::NBOX; ++b) {
                tc::tma_load_2d(sbase + C::K_OFF + b * C::BOX_BYTES, &tm_k, bar(B_KVFULL), b * 64, bh * L + k0);
                tc::tma_load_2d(sbase + C::V_OFF + b * C::BOX_BYTES, &tm_v, bar(B_KVFULL), b * 64, bh * L + k0);
            }
            int lastQ = -1, lastO = -1;
            // the loads in the order the MMA issuer consumes them: with two Q stages S_{i+1}
            // comes first (Q_{i+1}'s stage was freed by dK_{i-1}) and dO_{i+1} waits for dV_i;
            // with one, dV_i frees dO's stage before dK_i frees Q's
            auto load_q = [&](int i, int row) -> bool {
                const int sq = i % C::NSQ, uq = i / C::NSQ;
                if (uq > 0 && !tc::mbar_wait(bar(B_QEMPTY + sq), (uq - 1) & 1, aborted, status, kWaitLimitCycles))
                    return false;
                tc::mbar_expect_tx(bar(B_QFULL + sq), C::TILE_BYTES);
                for (int b = 0; b < C::NBOX; ++b)
                    tc::tma_load_2d(sbase + C::Q_OFF + sq * C::TILE_BYTES + b * C::BOX_BYTES, &tm_q,
                                    bar(B_QFULL + sq), b * 64, row);
                lastQ = i;
                return true;
            };
            auto load_do = [&](int i, int row) -> bool {
                const int so = i % C::NSO, uo = i / C::NSO;
                if (uo > 0 && !tc::mbar_wait(bar(B_DOEMPTY + so), (uo - 1) & 1, aborted, status, kWaitLimitCycles))
                    return false;
                tc::mbar_expect_tx(bar(B_DOFULL + so), C::TILE_BYTES);
                for (int b = 0; b < C::NBOX; ++b)
                    tc::tma_load_2d(sbase + C::DO_OFF + so * C::TILE_BYTES + b * C::BOX_BYTES, &tm_do,
                                    bar(B_DOFULL + so), b * 64, row);
                lastO = i;
                return true;
            };
            for (int i = 0; i < NQT; ++i) {
                const int row = bh * L + i * C::NQ;
                if (kEarlyS) {
                    if (!load_q(i, row) || !load_do(i, row)) break;
                } else {
                    if (!load_do(i, row) || !load_q(i, row)) break;
                }
            }
            if (aborted) {
                bool a2 = false;
                tc::mbar_wait(bar(B_KVFULL), 0, a2, status, kWaitLimitCycles);
                for (int i = (lastQ - C::NSQ + 1 > 0 ? lastQ - C::NSQ + 1 : 0); i <= lastQ; ++i) {
                    a2 = false;
                    tc::mbar_wait(bar(B_QFULL + i % C::NSQ), (i / C::NSQ) & 1, a2, status, kWaitLimitCycles);
                }
                for (int i = (lastO - C::NSO + 1 > 0 ? lastO - C::NSO + 1 : 0); i <= lastO; ++i) {
                    a2 = false;
                    tc::mbar_wait(bar(B_DOFULL + i % C::NSO), (i / C::NSO) & 1, a2, status, kWaitLimitCycles);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint64_t kdesc = tc::sdesc_sw128(sbase + C::K_OFF, 16, 1024);
            const uint64_t vdesc = tc::sdesc_sw128(sbase + C::V_OFF, 16, 1024);
            const uint64_t qdesc0 = tc::sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
            const uint64_t dodesc0 = tc::sdesc_sw128(sbase + C::DO_OFF, 16, 1024);
            const uint64_t qmn0 = tc::sdesc_sw128(sbase + C::Q_OFF, C::BOX_BYTES, 1024);   // Q as MN-major B
            const uint64_t domn0 = tc::sdesc_sw128(sbase + C::DO_OFF, C::BOX_BYTES, 1024); // dO as MN-major B
            const uint64_t pmn = tc::sdesc_sw128(sbase + C::P_OFF, C::BOX_BYTES, 1024);    // P as MN-major A
            const uint64_t dsmn = tc::sdesc_sw128(sbase + C::DS_OFF, C::BOX_BYTES, 1024);  // dS as MN-major A
            constexpr uint64_t kTileStep = C::TILE_BYTES >> 4;
            auto issue_s = [&](int st) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
                    tc::mma_ss(tmem, qdesc0 + st * kTileStep + off, kdesc + off, IDESC_S, kk > 0);
                }
            };
            auto issue_g = [&](int st) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
                    tc::mma_ss(tmem + C::G_COL, dodesc0 + st * kTileStep + off, vdesc + off, IDESC_S, kk > 0);
                }
            };
            // D[dcol] (+)= A^T-tile (keys x queries, MN-major) x B-tile (queries x d, MN-major); K-dim = 128 queries
            auto issue_kv = [&](uint32_t dcol, uint64_t adesc, uint64_t bdesc, bool first) {
#pragma unroll
                for (int kk = 0; kk < C::NQ / 16; ++kk) {
                    const uint64_t off = (uint64_t)((kk * 16 * 128) >> 4);  // 16 query rows further
                    tc::mma_ss(tmem + dcol, adesc + off, bdesc + off, IDESC_KV, (first && kk == 0) ? 0u : 1u);
                }
            };
            // S_i into the S columns (Q stage i % NSQ) once the softmax holds S_{i-1}; G_i likewise
            auto put_s = [&](int i) -> bool {
                if (i > 0 && !tc::mbar_wait(bar(B_SFREE), (i - 1) & 1, aborted, status, kWaitLimitCycles)) return false;
                const int sq = i % C::NSQ, uq = i / C::NSQ;
                if (!tc::mbar_wait(bar(B_QFULL + sq), uq & 1, aborted, status, kWaitLimitCycles)) return false;
                tc::fence_after_sync();
                issue_s(sq);
                tc::mma_commit(bar(B_SFULL));
                return true;
            };
            auto put_g = [&](int i) -> bool {
                if (i > 0 && !tc::mbar_wait(bar(B_GFREE), (i - 1) & 1, aborted, status, kWaitLimitCycles)) return false;
                const int so = i % C::NSO, uo = i / C::NSO;
                if (!tc::mbar_wait(bar(B_DOFULL + so), uo & 1, aborted, status, kWaitLimitCycles)) return false;
                tc::fence_after_sync();
                issue_g(so);
                tc::mma_commit(bar(B_GFULL));
                return true;
            };
            bool ok = tc::mbar_wait(bar(B_KVFULL), 0, aborted, status, kWaitLimitCycles);
            ok = ok && put_s(0) && put_g(0);
            for (int i = 0; ok && i < NQT; ++i) {
                const int sq = i % C::NSQ, so = i % C::NSO;
                const bool more = i + 1 < NQT;
                if (kEarlyS && more && !put_s(i + 1)) break;
                // dV_i once P_i is written
                if (!tc::mbar_wait(bar(B_PREADY), i & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                issue_kv(C::DV_COL, pmn, domn0 + so * kTileStep, i == 0);
                tc::mma_commit(bar(B_DOEMPTY + so));
                tc::mma_commit(bar(B_PFREE));
                if (kEarlyG && more && !put_g(i + 1)) break;
                // dK_i once dS_i is written
                if (!tc::mbar_wait(bar(B_DSREADY), i & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                issue_kv(C::DK_COL, dsmn, qmn0 + sq * kTileStep, i == 0);
                tc::mma_commit(bar(B_QEMPTY + sq));
                tc::mma_commit(bar(B_DSFREE));
                if (!kEarlyS && more && !put_s(i + 1)) break;
                if (!kEarlyG && more && !put_g(i + 1)) break;
            }
            if (!aborted) tc::mma_commit(bar(B_DKVFULL));
            tc::mma_commit(bar(B_DONE));
            bool a2 = false;
            tc::mbar_wait(bar(B_DONE), 0, a2, status, kWaitLimitCycles);
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int quarter = warp % 4;
        const int half = (warp - 2) / 4;
        const int r = quarter * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const float ln_b = logf((float)BS);
        const int jb = (k0 + 64 * half) / BS;  // this half's block
        uint8_t* ptile = smem + C::P_OFF;
        uint8_t* dstile = smem + C::DS_OFF;
        float* xch = reinterpret_cast<float*>(smem + C::XCH_OFF);
        // B = 128: add the other half's two sums (exchange ex of this tile, 0 or 1)
        auto exchange = [&](float2 mine, int ex) -> float2 {
            float2* slot = reinterpret_cast<float2*>(xch + (((ex * 2 + half) * 128) + r) * 2);
            *slot = mine;
            tc::mbar_arrive(bar(B_PAIR + quarter));
            if (!tc::mbar_wait_warp(bar(B_PAIR + quarter), ex, aborted, status, kWaitLimitCycles)) return mine;
            // the phase is complete (lane 0 saw it); each thread's own test of it is its acquire
            (void)tc::mbar_try_wait(bar(B_PAIR + quarter), ex);
            const float2 o = *reinterpret_cast<const float2*>(xch + (((ex * 2 + (1 - half)) * 128) + r) * 2);
            return make_float2(mine.x + o.x, mine.y + o.y);
        };
        for (int i = 0; i < NQT; ++i) {
            const int qrow = i * C::NQ + r;
            const bool valid = qrow < L;
            const int qt = (valid ? qrow : L - 1) / BS;
            const uint32_t* mrow = mask + ((size_t)bh * nblk + qt) * words;
            const float lse2 = valid ? __ldg(lse + (size_t)bh * L + qrow) * LOG2E : __int_as_float(0x7f800000);
            const float del = valid ? __ldg(delta + (size_t)bh * L + qrow) : 0.f;
            const bool sel = (__ldg(mrow + (jb >> 5)) >> (jb & 31)) & 1u;
            const float wp = (ORDER == 3) ? __ldg(wmat + ((size_t)bh * nblk + qt) * nblk + jb) : 0.f;
            // ---- pass 1: S alone -> P
            if (!tc::mbar_wait_warp(bar(B_SFULL), i & 1, aborted, status, kWaitLimitCycles)) break;
            tc::fence_after_sync();
            uint32_t xa[32], xb[32];
            tc::tmem_ld32(lane_base + 64 * half, xa);
            tc::tmem_ld32(lane_base + 64 * half + 32, xb);
            uint32_t x0raw = 0u;
            if (BS == 128 && half == 1) x0raw = tc::tmem_ld1(lane_base);  // the block's first logit
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_SFREE));
            const float x0 = (BS == 128 && half == 1) ? __uint_as_float(x0raw) : __uint_as_float(xa[0]);
            float2 ls = half_logit_sums(xa, xb, x0);
            if (BS == 128) ls = exchange(ls, 0);
            if (aborted) break;
            // the coefficients P needs: sb, w (gate held fixed), a = e^{l - lse}, Pu = c1 a
            float sb, a, A, X, Cc, Pu, inner;
            block_coefs<BS, ORDER>(x0, ls.x, ls.y, 0.f, 0.f, lse2, del, gate, ln_b, wp, sb, a, A, X, Cc, Pu, inner);
            if (i > 0 && !tc::mbar_wait_warp(bar(B_PFREE), (i - 1) & 1, aborted, status, kWaitLimitCycles)) break;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t pp[16];
                chunk_p(ch == 0 ? xa : xb, sel, lse2, sb, a, Pu, pp);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_swz16(ptile, r, 8 * half + 4 * ch + c,
                             make_uint4(pp[4 * c], pp[4 * c + 1], pp[4 * c + 2], pp[4 * c + 3]));
            }
            tc::fence_proxy_async_smem();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_PREADY));
            // ---- pass 2: G -> dS
            if (!tc::mbar_wait_warp(bar(B_GFULL), i & 1, aborted, status, kWaitLimitCycles)) break;
            tc::fence_after_sync();
            uint32_t ga[32], gb[32];
            tc::tmem_ld32(lane_base + C::G_COL + 64 * half, ga);
            tc::tmem_ld32(lane_base + C::G_COL + 64 * half + 32, gb);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_GFREE));
            float2 gsum = half_g_sums(xa, xb, ga, gb, x0);
            if (BS == 128) gsum = exchange(gsum, 1);
            if (aborted) break;
            block_coefs<BS, ORDER>(x0, ls.x, ls.y, gsum.x, gsum.y, lse2, del, gate, ln_b, wp, sb, a, A, X, Cc, Pu,
                                   inner);
            if (i > 0 && !tc::mbar_wait_warp(bar(B_DSFREE), (i - 1) & 1, aborted, status, kWaitLimitCycles)) break;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t dd[16];
                chunk_ds(ch == 0 ? xa : xb, ch == 0 ? ga : gb, sel, lse2, del, sb, A, X, Cc, dd);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_swz16(dstile, r, 8 * half + 4 * ch + c,
                             make_uint4(dd[4 * c], dd[4 * c + 1], dd[4 * c + 2], dd[4 * c + 3]));
            }
            tc::fence_proxy_async_smem();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_DSREADY));
        }
        // epilogue: this warp's column half of the dK and dV rows (TMEM lane = key) to global
        if (tc::mbar_wait_warp(bar(B_DKVFULL), 0, aborted, status, kWaitLimitCycles)) {
            tc::fence_after_sync();
            const int key = k0 + r;
            float* krow = dk + ((size_t)bh * L + key) * D + half * (D / 2);
            float* vrow = dv + ((size_t)bh * L + key) * D + half * (D / 2);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float* dst_row = part == 0 ? krow : vrow;
                const uint32_t col = (part == 0 ? C::DK_COL : C::DV_COL) + half * (D / 2);
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t raw[32];
                    tc::tmem_ld32(lane_base + col + c * 32, raw);
                    tc::tmem_wait_ld();
                    float4* dst = reinterpret_cast<float4*>(dst_row + c * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(__uint_as_float(raw[4 * e]), __uint_as_float(raw[4 * e + 1]),
                                             __uint_as_float(raw[4 * e + 2]), __uint_as_float(raw[4 * e + 3]));
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// The pooled w's gradient into dq and dk (after the dq and dk/dv kernels).  With W_ij the
// sum over query tile i's rows of dL/dl_tj (wpart, per 32 rows) on the blocks whose w was
// kept (wmat > 0), w_ij = 1/2 sum_c q2_ic var_jc gives
//   dq_mc += q_mc u_ic / B,   u_ic = sum_j W_ij var_jc          (rows m of tile i)
//   dk_nc += (k_nc - kbar_jc) z_jc / B,  z_jc = sum_i W_ij q2_ic  (keys n of block j)
// Every sum runs in a fixed order, so the result is the same on every run.
// bwd_pooled_dq_kernel: one CTA per (tile i, bh), 128 threads; also writes W (wsum).
template <int D, int BS>
__global__ void __launch_bounds__(128) bwd_pooled_dq_kernel(const bf16* __restrict__ q, const float* __restrict__ wmat,
                                                            const float* __restrict__ wpart,
                                                            const float* __restrict__ var, float* __restrict__ wsum,
                                                            float* __restrict__ dq, int L, int nblk) {
    extern __shared__ float ws_row[];  // [nblk]
    const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    constexpr int CPT = BS / 32;  // 32-row chunks per query tile
    const float* wr = wmat + ((size_t)bh * nblk + i) * nblk;
    for (int j = tid; j < nblk; j += 128) {
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < CPT; ++c) s += wpart[((size_t)bh * (L / 32) + i * CPT + c) * nblk + j];
        s = wr[j] > 0.f ? s : 0.f;
        ws_row[j] = s;
        wsum[((size_t)bh * nblk + i) * nblk + j] = s;
    }
    __syncthreads();
    if (tid >= D) return;
    float u = 0.f;
    const float* vb = var + (size_t)bh * nblk * D + tid;
    for (int j = 0; j < nblk; ++j) u = fmaf(ws_row[j], vb[(size_t)j * D], u);
    u *= 1.0f / (float)BS;
    for (int m = 0; m < BS; ++m) {
        const size_t e = ((size_t)bh * L + (size_t)i * BS + m) * D + tid;
        dq[e] = fmaf(__bfloat162float(q[e]), u, dq[e]);
    }
}

// bwd_pooled_dk_kernel: one CTA per (block j, bh), 128 threads.
template <int D, int BS>
__global__ void __launch_bounds__(128) bwd_pooled_dk_kernel(const bf16* __restrict__ k, const float* __restrict__ kbar,
                                                            const float* __restrict__ wsum,
                                                            const float* __restrict__ q2, float* __restrict__ dk,
                                                            int L, int nblk) {
    const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    if (tid >= D) return;
    float z = 0.f;
    const float* wc = wsum + (size_t)bh * nblk * nblk + j;
    const float* qb = q2 + (size_t)bh * nblk * D + tid;
    for (int i = 0; i < nblk; ++i) z = fmaf(wc[(size_t)i * nblk], qb[(size_t)i * D], z);
    z *= 1.0f / (float)BS;
    const float kb = kbar[((size_t)bh * nblk + j) * D + tid];
    for (int n = 0; n < BS; ++n) {
        const size_t e = ((size_t)bh * L + (size_t)j * BS + n) * D + tid;
        dk[e] = fmaf(__bfloat162float(k[e]) - kb, z, dk[e]);
    }
}

}  // namespace bwdtc
}  // namespace pisa
