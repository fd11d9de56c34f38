// Piecewise sparse attention on tcgen05 tensor cores (token form).
//
// What it computes (PISA paper, section 3.2 "Formulation"; "Sparse Linear
// Attention" blog, sections "Sparse Linear Attention" and "Going Further:
// Adding the Second-Order Term (PWT)"): for query row t of tile i and key block
// j, with x_n = q_t.k_{j,n} and s-bar = q_t.kbar_j = mean_n x_n,
//   j in S_i :  weights e^{x_n}                                (exact)
//   j in U_i :  weights e^{l}(1 + x_n - s-bar),  l = s-bar + w  (order >= 1)
//               weights e^{l}                                  (order 0)
//               denominator mass B e^{l}
//   w = 1/2 q^T C_j q = (1/2B) sum_n (x_n - s-bar)^2 for order 2 (0 above ln B
//   when gated), 0 otherwise.
// Summing e^{l}(1 + x_n - s-bar) v_n over the block gives exactly the paper's
// e^{l}(vsum_j + H_j q_t): the first-order numerator of the unselected block is
// evaluated through the block's tokens instead of the d x d statistic H_j.
// When d = 2B the two associations cost the same per (query, block), and this
// one needs no H_j stream and yields w from the same logits.  Both branches
// share one running max and one denominator (one online softmax).
//
// Structure (one CTA = 256 query rows of one (batch, head) = two 128-row M
// tiles; all key tiles of 128 keys are visited in order):
//   warp 0      TMA producer: Q once, then K and V tiles through NS stages
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2-5   softmax group 0 (M tile 0), warps 6-9 softmax group 1
// TMEM (512 columns): S0 | S1 | O0 | O1.  The softmax writes P (bf16) over the
// first half of its S columns and the PV MMA reads it from TMEM as operand A.
// MMA order per key tile jt: PV0(jt), S0(jt+1), PV1(jt), S1(jt+1), so each
// softmax group works while the tensor core runs the other group's products.
// P is handed over in two halves of 64 keys, each on its own barrier: the PV
// of the first half runs while the softmax computes the second.  Every MMA has
// N >= 128 (S: N = 128 keys; PV: N = d), the shapes at which tcgen05 with
// M = 128 runs at its full rate; N = 64 takes as long as N = 128.
// The running max is raised only when it grows by more than 2^8 (the output is
// rescaled then), so most tiles need no correction of O.
#pragma once

#include <cudaTypedefs.h>

#include <string>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace pisa {


template <int D>
struct TcCfg {
    static constexpr int NK = 128;                 // keys per tile
    static constexpr int MQ = 128;                 // rows per M tile
    static constexpr int NS = (D == 128) ? 2 : 4;  // K/V stages
    static constexpr int BOX = 64;                 // bf16 columns per 128-byte swizzle box
    static constexpr int NBOX = D / BOX;
    static constexpr uint32_t BOX_BYTES = 128 * 128;     // 128 rows x 128 bytes
    static constexpr uint32_t TILE_BYTES = NBOX * BOX_BYTES;
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t K_OFF = Q_OFF + 2 * TILE_BYTES;
    static constexpr uint32_t V_OFF = K_OFF + NS * TILE_BYTES;
    static constexpr uint32_t BAR_OFF = V_OFF + NS * TILE_BYTES;
    // QFULL; KFULL, KEMPTY, VFULL, VEMPTY per stage; SFULL, PHALF, PFULL, OFULL
    // per M tile; DONE
    static constexpr uint32_t NBAR = 1 + 4 * NS + 2 + 2 + 2 + 2 + 1;
    static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;  // + alignment slack
    static constexpr uint32_t O_COL0 = 256;
    static constexpr uint32_t TMEM_COLS = 512;
};

// Pass 1 over the N logits of one key block (fp32 bits in x): returns the
// block's candidate for the running max in log2 units.  Selected block: its
// largest logit.  Unselected block: l = s-bar + w, with s-bar = mean of the
// logits (= q.kbar_j) and w the second-order mass term (ORDER 2: from the
// logits' spread, gated at ln B; ORDER 3: the pooled value w_pool); sbar and
// l2 = l log2 e are returned too.  Reductions run on packed fp32 pairs in four
// independent chains.
template <int N, int ORDER>
__device__ __forceinline__ float block_pass1(const uint32_t* x, bool sel, int gate, float ln_b, float w_pool,
                                             float& sbar, float& l2) {
    constexpr float LOG2E = 1.4426950408889634f;
    if (sel) {
        float m4[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) m4[a] = fmaxf(__uint_as_float(x[2 * a]), __uint_as_float(x[2 * a + 1]));
#pragma unroll
        for (int e = 8; e < N; e += 8)
#pragma unroll
            for (int a = 0; a < 4; ++a)
                m4[a] = tc::max3(m4[a], __uint_as_float(x[e + 2 * a]), __uint_as_float(x[e + 2 * a + 1]));
        sbar = 0.f;
        l2 = 0.f;
        return tc::max3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * LOG2E;
    }
    uint64_t s2[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) s2[a] = tc::f2_make(__uint_as_float(x[2 * a]), __uint_as_float(x[2 * a + 1]));
#pragma unroll
    for (int e = 8; e < N; e += 8)
#pragma unroll
        for (int a = 0; a < 4; ++a)
            s2[a] = tc::f2_add(s2[a], tc::f2_make(__uint_as_float(x[e + 2 * a]), __uint_as_float(x[e + 2 * a + 1])));
    constexpr float inv_n = 1.0f / (float)N;
    const float2 st = tc::f2_split(tc::f2_add(tc::f2_add(s2[0], s2[1]), tc::f2_add(s2[2], s2[3])));
    const float sb = (st.x + st.y) * inv_n;
    float w = 0.f;
    if (ORDER == 2) {
        // second pass over the deviations x_n - s-bar: a sum of squares, so w >= 0 as the
        // pages have it (Jensen), and no cancellation when |s-bar| is large against the spread
        const uint64_t negs = tc::f2_make(-sb, -sb);
        uint64_t q2[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const uint64_t t = tc::f2_add(tc::f2_make(__uint_as_float(x[2 * a]), __uint_as_float(x[2 * a + 1])), negs);
            q2[a] = tc::f2_mul(t, t);
        }
#pragma unroll
        for (int e = 8; e < N; e += 8)
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const uint64_t t = tc::f2_add(
                    tc::f2_make(__uint_as_float(x[e + 2 * a]), __uint_as_float(x[e + 2 * a + 1])), negs);
                q2[a] = tc::f2_fma(t, t, q2[a]);
            }
        const float2 qq = tc::f2_split(tc::f2_add(tc::f2_add(q2[0], q2[1]), tc::f2_add(q2[2], q2[3])));
        w = 0.5f * (qq.x + qq.y) * inv_n;
        if (gate && w > ln_b) w = 0.f;
    } else if (ORDER == 3) {
        w = w_pool;
    }
    sbar = sb;
    l2 = (sb + w) * LOG2E;
    return l2;
}

// Pass 2 over 32 logits of one block: the bf16 weights as 16 packed pairs.
// Selected: e^{x - m} (every fourth exponential on the FMA pipe); returns their
// sum for the denominator.  Unselected: alpha x + c0 with alpha = e^{l - m} and
// c0 = alpha (1 - s-bar) (ORDER >= 1), or alpha (ORDER 0); returns 0 (the
// block's mass B alpha is added once per block by the caller).
template <int ORDER>
__device__ __forceinline__ float chunk_pass2(const uint32_t* x, bool sel, float m_run, float alpha, float c0,
                                             uint32_t (&pk)[16]) {
    constexpr float LOG2E = 1.4426950408889634f;
    if (sel) {
        const uint64_t negm = tc::f2_make(-m_run, -m_run), log2e2 = tc::f2_make(LOG2E, LOG2E);
        uint64_t d2[2] = {tc::f2_make(0.f, 0.f), tc::f2_make(0.f, 0.f)};
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float2 t = tc::f2_split(
                tc::f2_fma(tc::f2_make(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), log2e2, negm));
            const float a0 = tc::ex2(t.x);
            const float a1 = (e & 1) ? tc::ex2_fma(t.y) : tc::ex2(t.y);
            d2[e & 1] = tc::f2_add(d2[e & 1], tc::f2_make(a0, a1));
            pk[e] = tc::pack_bf16x2(a0, a1);
        }
        const float2 dd = tc::f2_split(tc::f2_add(d2[0], d2[1]));
        return dd.x + dd.y;
    }
    if (ORDER >= 1) {
        const uint64_t al2 = tc::f2_make(alpha, alpha), c02 = tc::f2_make(c0, c0);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float2 wv = tc::f2_split(
                tc::f2_fma(al2, tc::f2_make(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), c02));
            pk[e] = tc::pack_bf16x2(wv.x, wv.y);
        }
    } else {
        const uint32_t a2 = tc::pack_bf16x2(alpha, alpha);
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = a2;
    }
    return 0.f;
}

template <int D, int BS, int ORDER>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const uint32_t* __restrict__ mask, bf16* __restrict__ out,
                   int L, int nblk, int words, int gate, float ln_b, const float* __restrict__ wmat,
                   unsigned* status, float* __restrict__ lse) {
    // ORDER: 0 zeroth, 1 first, 2 first + exact w from the logits, 3 first + the
    // pooled diagonal w of wmat ([BH, nblk, nblk], row = query tile, already gated)
    using C = TcCfg<D>;
    // with two K/V stages the producer frees stages off group 1's S-full
    // barrier, and the MMA thread issues no empty-barrier commits (each
    // tcgen05.commit in the stream stalls the tensor pipe for tens of cycles)
    constexpr bool kSfullRelease = (C::NS == 2);
    constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, false);  // S = Q K^T, N = 128 keys
    constexpr uint32_t IDESC_O = tc::idesc_bf16(128, D, true);     // O += P V, N = d, V MN-major

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_addr(smem);
    uint64_t* bars = (uint64_t*)(smem + C::BAR_OFF);
    uint32_t* tmem_slot = (uint32_t*)(bars + C::NBAR);
    auto bar = [&](int i) { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
    const int B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 1 + C::NS, B_VFULL = 1 + 2 * C::NS, B_VEMPTY = 1 + 3 * C::NS;
    const int B_SFULL = 1 + 4 * C::NS, B_PHALF = B_SFULL + 2, B_PFULL = B_PHALF + 2, B_OFULL = B_PFULL + 2;
    const int B_DONE = B_OFULL + 2;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = blockIdx.y;
    const int q0 = blockIdx.x * 256;
    const int NT = L / C::NK;
    bool aborted = false;

    if (threadIdx.x == 0) {
        tc::mbar_init(bar(B_QFULL), 1);
        for (int s = 0; s < C::NS; ++s) {
            tc::mbar_init(bar(B_KFULL + s), 1);
            tc::mbar_init(bar(B_KEMPTY + s), 1);
            tc::mbar_init(bar(B_VFULL + s), 1);
            tc::mbar_init(bar(B_VEMPTY + s), 1);
        }
        for (int h = 0; h < 2; ++h) {
            tc::mbar_init(bar(B_SFULL + h), 1);
            tc::mbar_init(bar(B_PHALF + h), 128);
            tc::mbar_init(bar(B_PFULL + h), 128);
            tc::mbar_init(bar(B_OFULL + h), 1);
        }
        tc::mbar_init(bar(B_DONE), 1);
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
            const int row0 = bh * L + q0;
            tc::mbar_expect_tx(bar(B_QFULL), 2 * C::TILE_BYTES);
            for (int h = 0; h < 2; ++h)
                for (int b = 0; b < C::NBOX; ++b)
                    tc::tma_load_2d(sbase + C::Q_OFF + h * C::TILE_BYTES + b * C::BOX_BYTES, &tm_q, bar(B_QFULL),
                                    b * C::BOX, row0 + h * C::MQ);
            int lastK = -1, lastV = -1;
            for (int jt = 0; jt < NT; ++jt) {
                const int st = jt % C::NS, u = jt / C::NS;
                if (kSfullRelease) {
                    // two stages: S1(jt-1) completing (group 1's S-full barrier) means
                    // S0/S1(jt-2) and PV1(jt-2) are done, so the K and V stage of tile
                    // jt-2 are free.  One wait per tile, phases in order; S1(jt) needs
                    // K(jt), not loaded yet, so the barrier is never two phases ahead.
                    if (jt >= 1 && !tc::mbar_wait(bar(B_SFULL + 1), (jt - 1) & 1, aborted, status, kWaitLimitCycles))
                        break;
                } else if (u > 0 &&
                           !tc::mbar_wait(bar(B_KEMPTY + st), (u - 1) & 1, aborted, status, kWaitLimitCycles)) {
                    break;
                }
                tc::mbar_expect_tx(bar(B_KFULL + st), C::TILE_BYTES);
                for (int b = 0; b < C::NBOX; ++b)
                    tc::tma_load_2d(sbase + C::K_OFF + st * C::TILE_BYTES + b * C::BOX_BYTES, &tm_k,
                                    bar(B_KFULL + st), b * C::BOX, bh * L + jt * C::NK);
                lastK = jt;
                if (!kSfullRelease && u > 0 &&
                    !tc::mbar_wait(bar(B_VEMPTY + st), (u - 1) & 1, aborted, status, kWaitLimitCycles))
                    break;
                tc::mbar_expect_tx(bar(B_VFULL + st), C::TILE_BYTES);
                for (int b = 0; b < C::NBOX; ++b)
                    tc::tma_load_2d(sbase + C::V_OFF + st * C::TILE_BYTES + b * C::BOX_BYTES, &tm_v,
                                    bar(B_VFULL + st), b * C::BOX, bh * L + jt * C::NK);
                lastV = jt;
            }
            if (aborted) {
                // let every copy already issued land before the CTA exits
                bool a2 = false;
                tc::mbar_wait(bar(B_QFULL), 0, a2, status, kWaitLimitCycles);
                for (int jt = (lastK - C::NS + 1 > 0 ? lastK - C::NS + 1 : 0); jt <= lastK; ++jt) {
                    a2 = false;
                    tc::mbar_wait(bar(B_KFULL + jt % C::NS), (jt / C::NS) & 1, a2, status, kWaitLimitCycles);
                }
                for (int jt = (lastV - C::NS + 1 > 0 ? lastV - C::NS + 1 : 0); jt <= lastV; ++jt) {
                    a2 = false;
                    tc::mbar_wait(bar(B_VFULL + jt % C::NS), (jt / C::NS) & 1, a2, status, kWaitLimitCycles);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            // descriptors of the operand bases; a K-step adds its byte offset >> 4
            // to the start-address field (addresses stay below 2^18)
            const uint64_t qdesc0 = tc::sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
            const uint64_t kdesc0 = tc::sdesc_sw128(sbase + C::K_OFF, 16, 1024);
            const uint64_t vdesc0 = tc::sdesc_sw128(sbase + C::V_OFF, C::BOX_BYTES, 1024);
            constexpr uint64_t kTileStep = C::TILE_BYTES >> 4;  // one tile further in shared memory
            auto issue_s = [&](int h, int st) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
                    tc::mma_ss(tmem + (uint32_t)(h * 128), qdesc0 + h * kTileStep + off, kdesc0 + st * kTileStep + off,
                               IDESC_S, kk > 0);
                }
            };
            // PV over one half of the key tile (keys 64*half .. 64*half + 63)
            auto issue_pv = [&](int h, int st, int half, bool first) {
#pragma unroll
                for (int kk = half * 4; kk < half * 4 + 4; ++kk) {
                    tc::mma_ts(tmem + C::O_COL0 + h * D, tmem + (uint32_t)(h * 128) + kk * 8,
                               vdesc0 + st * kTileStep + (uint64_t)((kk * 16 * 128) >> 4), IDESC_O, (first && kk == 0) ? 0u : 1u);
                }
            };
            bool ok = tc::mbar_wait(bar(B_QFULL), 0, aborted, status, kWaitLimitCycles);
            ok = ok && tc::mbar_wait(bar(B_KFULL + 0), 0, aborted, status, kWaitLimitCycles);
            if (ok) {
                issue_s(0, 0);
                tc::mma_commit(bar(B_SFULL + 0));
                issue_s(1, 0);
                tc::mma_commit(bar(B_SFULL + 1));
                if (!kSfullRelease) tc::mma_commit(bar(B_KEMPTY + 0));
            }
            for (int jt = 0; ok && jt < NT; ++jt) {
                const int st = jt % C::NS, u = jt / C::NS;
                const int st1 = (jt + 1) % C::NS, u1 = (jt + 1) / C::NS;
                const bool more = jt + 1 < NT;
                if (!tc::mbar_wait(bar(B_VFULL + st), u & 1, aborted, status, kWaitLimitCycles)) break;
                if (!tc::mbar_wait(bar(B_PHALF + 0), jt & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                issue_pv(0, st, 0, jt == 0);
                if (!tc::mbar_wait(bar(B_PFULL + 0), jt & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                issue_pv(0, st, 1, false);
                if (!more) tc::mma_commit(bar(B_OFULL + 0));
                if (more) {
                    if (!tc::mbar_wait(bar(B_KFULL + st1), u1 & 1, aborted, status, kWaitLimitCycles)) break;
                    issue_s(0, st1);
                    tc::mma_commit(bar(B_SFULL + 0));
                }
                if (!tc::mbar_wait(bar(B_PHALF + 1), jt & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                issue_pv(1, st, 0, jt == 0);
                if (!tc::mbar_wait(bar(B_PFULL + 1), jt & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                issue_pv(1, st, 1, false);
                if (!more) tc::mma_commit(bar(B_OFULL + 1));
                if (!kSfullRelease) tc::mma_commit(bar(B_VEMPTY + st));
                if (more) {
                    issue_s(1, st1);
                    tc::mma_commit(bar(B_SFULL + 1));
                    if (!kSfullRelease) tc::mma_commit(bar(B_KEMPTY + st1));
                }
            }
            // every MMA issued by this thread has completed before TMEM is freed
            tc::mma_commit(bar(B_DONE));
            bool a2 = false;
            tc::mbar_wait(bar(B_DONE), 0, a2, status, kWaitLimitCycles);
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int h = (warp - 2) / 4;             // M tile of this group
        const int quarter = warp % 4;             // TMEM lane quarter of this warp
        const int r = quarter * 32 + lane;        // row inside the M tile = TMEM lane
        const int qrow = q0 + h * C::MQ + r;      // query row inside the head
        const bool valid = qrow < L;
        int qt = (qrow < L ? qrow : L - 1) / BS;  // query tile (selection row)
        const uint32_t* mrow = mask + ((size_t)bh * nblk + qt) * words;
        const float* wrow = (ORDER == 3) ? wmat + ((size_t)bh * nblk + qt) * nblk : nullptr;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t s_addr = lane_base + (uint32_t)(h * 128);
        const uint32_t o_addr = lane_base + C::O_COL0 + h * D;
        constexpr int BPT = C::NK / BS;           // blocks per key tile
        float m_run = -INFINITY;                  // running max (log2 units)
        float dsum = 0.f;                         // denominator (scaled by 2^-m_run)
        int mword_idx = -1;                       // cached selection-mask word
        uint32_t mword = 0u;

        for (int jt = 0; jt < NT; ++jt) {
            if (!tc::mbar_wait_warp(bar(B_SFULL + h), jt & 1, aborted, status, kWaitLimitCycles)) break;
            tc::fence_after_sync();
            bool sel[BPT];
            float wp[BPT];
            if (((jt * BPT) >> 5) != mword_idx) {
                mword_idx = (jt * BPT) >> 5;
                mword = __ldg(mrow + mword_idx);
            }
#pragma unroll
            for (int b = 0; b < BPT; ++b) {
                const int j = jt * BPT + b;  // the BPT blocks of a tile share one mask word
                sel[b] = (mword >> (j & 31)) & 1u;
                wp[b] = (ORDER == 3 && !sel[b]) ? __ldg(wrow + j) : 0.f;
            }
            // the whole 128-column S tile in registers: one TMEM round trip per
            // tile, and pass 2 reuses the values
            uint32_t sv[C::NK];
#pragma unroll
            for (int c = 0; c < C::NK / 32; ++c)
                tc::tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32 * c));
            tc::tmem_wait_ld();
            // pass 1: per-block statistic of the logits
            float cand[BPT], sbar[BPT], l2[BPT];
#pragma unroll
            for (int b = 0; b < BPT; ++b)
                cand[b] = block_pass1<BS, ORDER>(sv + b * BS, sel[b], gate, ln_b, wp[b], sbar[b], l2[b]);
            float mc = cand[0];
#pragma unroll
            for (int b = 1; b < BPT; ++b) mc = fmaxf(mc, cand[b]);
            // raise the running max only when it grows by more than 2^8; the
            // decision is per row, the O correction is done by the whole warp
            const bool raise = mc > m_run + 8.0f;
            const float scale = raise ? tc::ex2(m_run - mc) : 1.0f;
            if (raise) {
                dsum *= scale;
                m_run = mc;
            }
            if (__any_sync(0xffffffffu, raise) && jt > 0) {
                // the previous PV of this tile is complete (covered by S_FULL)
#pragma unroll 1
                for (int c = 0; c < D / 16; ++c) {
                    uint32_t raw[16];
                    tc::tmem_ld16(o_addr + c * 16, raw);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * scale);
                    tc::tmem_st16(o_addr + c * 16, raw);
                }
            }
            // coefficients of the Taylor blocks and their mass B e^{l}
            float alpha[BPT], c0[BPT];
#pragma unroll
            for (int b = 0; b < BPT; ++b) {
                alpha[b] = 0.f;
                c0[b] = 0.f;
                if (!sel[b]) {
                    alpha[b] = tc::ex2(l2[b] - m_run);
                    dsum = fmaf((float)BS, alpha[b], dsum);
                    c0[b] = alpha[b] * (1.0f - sbar[b]);
                }
            }
            // pass 2 in two halves of 64 keys: P (bf16, 32 packed columns per
            // half) goes over the S columns; each half is handed to the MMA
            // warp on its own barrier, so the first half's PV runs while the
            // second half is computed
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int col = half * 64 + c * 32;  // first key of this chunk
                    const int b = col / BS;
                    uint32_t pk[16];
                    dsum += chunk_pass2<ORDER>(sv + col, sel[b], m_run, alpha[b], c0[b], pk);
                    tc::tmem_st16(s_addr + col / 2, pk);
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
                tc::mbar_arrive(bar((half == 0 ? B_PHALF : B_PFULL) + h));
            }
        }
        // epilogue: o = N / D
        if (tc::mbar_wait_warp(bar(B_OFULL + h), 0, aborted, status, kWaitLimitCycles)) {
            tc::fence_after_sync();
            const float inv = 1.0f / dsum;
            // optional log-denominator ln D_t = m ln 2 + ln(dsum) (m in log2 units), for the backward
            if (lse && valid) lse[(size_t)bh * L + qrow] = fmaf(m_run, 0.6931471805599453f, logf(dsum));
            bf16* orow = out + ((size_t)bh * L + (valid ? qrow : 0)) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t raw[32];
                tc::tmem_ld32(o_addr + c * 32, raw);
                tc::tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = tc::pack_bf16x2(__uint_as_float(raw[2 * e]) * inv, __uint_as_float(raw[2 * e + 1]) * inv);
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
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

inline bool attn_tc_supported(int d, int B) { return (d == 64 || d == 128) && (B == 64 || B == 128); }

// Host: build the tensor maps and launch.  Requires L % 128 == 0 (checked).
// order 3 = order 2 with the pooled w matrix `wmat` ([BH, nblk, nblk] fp32, gated).
inline pisa_status run_attn_tc(const void* q, const void* k, const void* v, const uint32_t* mask, void* out, long BH,
                               int L, int d, int B, int nblk, int words, int order, int gate, const float* wmat,
                               unsigned* status, cudaStream_t s, std::string* err, float* lse = nullptr) {
    if (L % 128) {
        *err = "tensor-core path needs L % 128 == 0";
        return PISA_ERR_UNSUPPORTED;
    }
    if (BH * (long)L > 0x7fffffffL) {
        *err = "tensor-core path needs batch*heads*L < 2^31";
        return PISA_ERR_UNSUPPORTED;
    }
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
    CUtensorMap maps[3];
    const void* ptrs[3] = {q, k, v};
    for (int t = 0; t < 3; ++t) {
        cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)(BH * L)};
        cuuint64_t gstride[1] = {(cuuint64_t)d * 2};
        cuuint32_t box[2] = {64, 128};
        cuuint32_t estride[2] = {1, 1};
        CUresult cr = encode(&maps[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptrs[t]), gdim, gstride,
                             box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS) {
            *err = "cuTensorMapEncodeTiled failed (" + std::to_string((int)cr) + ")";
            return PISA_ERR_CUDA;
        }
    }
    const float ln_b = logf((float)B);
    dim3 grid((unsigned)((L + 255) / 256), (unsigned)BH);
    cudaError_t e = cudaSuccess;
#define PISA_TC_LAUNCH(DD, BB, OO)                                                                             \
    if (d == DD && B == BB && order == OO) {                                                                   \
        auto kern = attn_tc_kernel<DD, BB, OO>;                                                                \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TcCfg<DD>::SMEM);     \
        if (e == cudaSuccess) {                                                                                \
            kern<<<grid, kTcThreads, TcCfg<DD>::SMEM, s>>>(maps[0], maps[1], maps[2], mask, (bf16*)out, L, nblk, \
                                                           words, gate, ln_b, wmat, status, lse);              \
            e = cudaGetLastError();                                                                            \
        }                                                                                                      \
    } else
    PISA_TC_LAUNCH(64, 64, 0)
    PISA_TC_LAUNCH(64, 64, 1)
    PISA_TC_LAUNCH(64, 64, 2)
    PISA_TC_LAUNCH(64, 64, 3)
    PISA_TC_LAUNCH(64, 128, 0)
    PISA_TC_LAUNCH(64, 128, 1)
    PISA_TC_LAUNCH(64, 128, 2)
    PISA_TC_LAUNCH(64, 128, 3)
    PISA_TC_LAUNCH(128, 64, 0)
    PISA_TC_LAUNCH(128, 64, 1)
    PISA_TC_LAUNCH(128, 64, 2)
    PISA_TC_LAUNCH(128, 64, 3)
    PISA_TC_LAUNCH(128, 128, 0)
    PISA_TC_LAUNCH(128, 128, 1)
    PISA_TC_LAUNCH(128, 128, 2)
    PISA_TC_LAUNCH(128, 128, 3) {
        *err = "no tensor-core kernel for this d/B/order";
        return PISA_ERR_UNSUPPORTED;
    }
#undef PISA_TC_LAUNCH
    if (e != cudaSuccess) {
        *err = std::string("attn_tc_kernel launch: ") + cudaGetErrorString(e);
        return PISA_ERR_CUDA;
    }
    return PISA_OK;
}

}  // namespace pisa
