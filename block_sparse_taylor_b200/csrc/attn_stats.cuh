// Statistics-form piecewise sparse attention on CUDA cores.
//
// For every query row t of tile i, one online softmax over the key blocks in
// index order:
//   j in S_i (selected): exact logits x = q_t.k_{j,n}, weights e^{x - m}
//   j in U_i (the rest): one virtual token with logit l = q_t.kbar_j + w,
//       mass B e^{l - m} in the denominator and e^{l - m}(vsum_j + H_j q_t) in
//       the numerator; w = 1/2 q_t^T C_j q_t for order 2 (0 above ln B with the
//       gate), 0 otherwise; the H_j term is dropped for order 0.
// PISA paper section 3.2 "Formulation" (shared denominator D_t), section 3.4
// phases 1-2; "Sparse Linear Attention" blog, sections "Sparse Linear
// Attention" (virtual token, first-order correction) and "Going Further:
// Adding the Second-Order Term (PWT)" (w, the shared corrected logit, the
// ln B gate).
//
// One CTA per (RQ query rows of a tile, bh), 8 warps; warp w owns rows w, w+8,
// ...; the running max, denominator and numerator of every row live in shared
// memory.  RQ = B, or B/2 when a whole tile's state does not fit (fp32, d = B = 128).
// The block being processed (K_j and V_j, or H_j and C_j) is staged in shared
// memory with padded rows so that lanes reading different rows hit different
// banks.  This is the fp32 path and the reference path for the tensor-core
// kernel; it is not the fast path for bf16.
#pragma once

#include "common.cuh"

namespace pisa {

template <typename T, int D, int BS, int RQ>
struct AttnStatsSmemRQ {
    static constexpr int QS = D + 1;                           // fp32 row stride
    static constexpr int XS = D + (sizeof(T) == 2 ? 2 : 1);    // T row stride (odd word count)
    static constexpr int ROWS = (BS > D ? BS : D);
    static constexpr size_t bytes = sizeof(float) * ((size_t)RQ * QS + (size_t)RQ * D + 2 * RQ + 2 * D) +
                                    sizeof(T) * 2 * (size_t)ROWS * XS;
};
// query rows per CTA: the whole tile when it fits in 227 KB of shared memory, else half
template <typename T, int D, int BS>
struct AttnStatsSmem {
    static constexpr int RQ = (AttnStatsSmemRQ<T, D, BS, BS>::bytes <= 227 * 1024) ? BS : BS / 2;
    static constexpr int QS = AttnStatsSmemRQ<T, D, BS, RQ>::QS;
    static constexpr int XS = AttnStatsSmemRQ<T, D, BS, RQ>::XS;
    static constexpr int ROWS = AttnStatsSmemRQ<T, D, BS, RQ>::ROWS;
    static constexpr size_t bytes = AttnStatsSmemRQ<T, D, BS, RQ>::bytes;
};

template <typename T, int D, int BS>
__global__ void __launch_bounds__(256) attn_stats_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const float* __restrict__ kbar, const float* __restrict__ vsum, const T* __restrict__ hstat,
    const T* __restrict__ cov, const uint32_t* __restrict__ mask, T* __restrict__ out, int L, int nblk,
    int words, int order, int gate, float ln_b, const float* __restrict__ wmat, float* __restrict__ lse) {
    // wmat (order 2, optional): PWT's pooled diagonal w per (query tile, block), gated
    using SM = AttnStatsSmem<T, D, BS>;
    constexpr int QS = SM::QS, XS = SM::XS, W = D / 32, RQ = SM::RQ;
    extern __shared__ __align__(16) float sm_attn[];
    float* qs = sm_attn;            // [RQ][QS]
    float* Ns = qs + RQ * QS;       // [RQ][D]
    float* ms = Ns + RQ * D;        // [RQ]
    float* ds = ms + RQ;            // [RQ]
    float* aux = ds + RQ;           // [2][D]: kbar_j, vsum_j
    T* st0 = (T*)(aux + 2 * D);     // [ROWS][XS]: K_j or H_j
    T* st1 = st0 + SM::ROWS * XS;   // [ROWS][XS]: V_j or C_j
    const int i = blockIdx.x / (BS / RQ), part = blockIdx.x % (BS / RQ), bh = blockIdx.y, tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32;
    const size_t base = ((size_t)bh * L + (size_t)i * BS + (size_t)part * RQ) * D;
    for (int e = tid; e < RQ * D; e += 256) {
        qs[(e / D) * QS + e % D] = to_f(q[base + e]);
        Ns[e] = 0.f;
    }
    for (int r = tid; r < RQ; r += 256) {
        ms[r] = -INFINITY;
        ds[r] = 0.f;
    }
    const uint32_t* mrow = mask + ((size_t)bh * nblk + i) * words;
    __syncthreads();

    for (int j = 0; j < nblk; ++j) {
        const bool sel = (mrow[j >> 5] >> (j & 31)) & 1u;
        if (sel) {
            const size_t kb = ((size_t)bh * L + (size_t)j * BS) * D;
            for (int e = tid; e < BS * D; e += 256) {
                st0[(e / D) * XS + e % D] = k[kb + e];
                st1[(e / D) * XS + e % D] = v[kb + e];
            }
        } else {
            const size_t so = ((size_t)bh * nblk + j) * D;
            for (int e = tid; e < D; e += 256) {
                aux[e] = kbar[so + e];
                aux[D + e] = vsum[so + e];
            }
            if (order >= 1) {
                const T* hj = hstat + so * D;
                for (int e = tid; e < D * D; e += 256) st0[(e / D) * XS + e % D] = hj[e];
            }
            if (order == 2 && !wmat) {
                const T* cj = cov + so * D;
                for (int e = tid; e < D * D; e += 256) st1[(e / D) * XS + e % D] = cj[e];
            }
        }
        __syncthreads();
        for (int r = warp; r < RQ; r += 8) {
            const float* qr = qs + r * QS;
            const float m_old = ms[r], d_old = ds[r];
            float acc[W];
#pragma unroll
            for (int w = 0; w < W; ++w) acc[w] = Ns[r * D + lane + 32 * w];
            if (sel) {
                constexpr int U = BS / 32;
                float x[U];
                float mx = -INFINITY;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const T* kr = st0 + (lane + 32 * u) * XS;
                    float s = 0.f;
                    for (int c = 0; c < D; ++c) s = fmaf(qr[c], to_f(kr[c]), s);
                    x[u] = s;
                    mx = fmaxf(mx, s);
                }
                mx = warp_max(mx);
                const float m_new = fmaxf(m_old, mx);
                const float scale = expf(m_old - m_new);
                float ps = 0.f;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    x[u] = expf(x[u] - m_new);
                    ps += x[u];
                }
                ps = warp_sum(ps);
#pragma unroll
                for (int w = 0; w < W; ++w) acc[w] *= scale;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    for (int n = 0; n < 32; ++n) {
                        const float p = __shfl_sync(0xffffffffu, x[u], n);
                        const T* vr = st1 + (32 * u + n) * XS;
#pragma unroll
                        for (int w = 0; w < W; ++w) acc[w] = fmaf(p, to_f(vr[lane + 32 * w]), acc[w]);
                    }
                }
                if (lane == 0) {
                    ms[r] = m_new;
                    ds[r] = d_old * scale + ps;
                }
            } else {
                float s = 0.f;
#pragma unroll
                for (int w = 0; w < W; ++w) s = fmaf(qr[lane + 32 * w], aux[lane + 32 * w], s);
                s = warp_sum(s);
                float wq = 0.f;
                if (order == 2 && wmat) {
                    wq = wmat[((size_t)bh * nblk + i) * nblk + j];
                } else if (order == 2) {
                    float part = 0.f;
#pragma unroll
                    for (int w = 0; w < W; ++w) {
                        const int a = lane + 32 * w;
                        const T* ca = st1 + a * XS;
                        float t = 0.f;
                        for (int b = 0; b < D; ++b) t = fmaf(to_f(ca[b]), qr[b], t);
                        part = fmaf(qr[a], t, part);
                    }
                    // C_j is PSD, so w >= 0 (Jensen); rounding of the stored C_j must not make it negative
                    wq = fmaxf(0.5f * warp_sum(part), 0.f);
                    if (gate && wq > ln_b) wq = 0.f;
                }
                const float l = s + wq;
                const float m_new = fmaxf(m_old, l);
                const float scale = expf(m_old - m_new);
                const float alpha = expf(l - m_new);
#pragma unroll
                for (int w = 0; w < W; ++w) {
                    const int a = lane + 32 * w;
                    float hq = 0.f;
                    if (order >= 1) {
                        const T* ha = st0 + a * XS;
                        for (int b = 0; b < D; ++b) hq = fmaf(to_f(ha[b]), qr[b], hq);
                    }
                    acc[w] = fmaf(acc[w], scale, alpha * (aux[D + a] + hq));
                }
                if (lane == 0) {
                    ms[r] = m_new;
                    ds[r] = fmaf(d_old, scale, (float)BS * alpha);
                }
            }
#pragma unroll
            for (int w = 0; w < W; ++w) Ns[r * D + lane + 32 * w] = acc[w];
            __syncwarp();
        }
        __syncthreads();
    }
    for (int e = tid; e < RQ * D; e += 256) out[base + e] = from_f<T>(Ns[e] / ds[e / D]);
    // optional log-denominator ln D_t = m + ln(D scaled by e^-m), for the backward
    if (lse)
        for (int r = tid; r < RQ; r += 256) lse[(size_t)bh * L + (size_t)i * BS + (size_t)part * RQ + r] = ms[r] + logf(ds[r]);
}

}  // namespace pisa
