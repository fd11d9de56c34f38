// PISA hybrid attention on tcgen05 tensor cores: exact selected blocks,
// zeroth-order virtual tokens for every other block, and the first-order term
// through the global statistic H-bar.
//
// What it computes (PISA paper, section 3.2 "Formulation", section 3.3
// "Global First-Order Correction", Figure 3 and section 3.4 phases 1-3; the
// "Sparse Linear Attention" blog, section "Sparse Linear Attention"): for query
// row t of tile i, with alpha_tj = e^{q_t . kbar_j},
//   D_t = sum_{j in S_i} sum_n e^{q.k_n} + sum_{j in U_i} B alpha_tj
//   N_t = sum_{j in S_i} sum_n e^{q.k_n} v_n + sum_{j in U_i} alpha_tj vsum_j
//         + [order 1] (sum_{j in U_i} alpha_tj) H-bar q_t
//   o_t = N_t / D_t,   H-bar = (B/L) sum_j H_j  (one d x d matrix per head).
//
// Work of one CTA (256 query rows = two 128-row M tiles of one (batch, head)):
//   1. union tiles: the blocks selected by any of the CTA's query tiles, in
//      ascending order, 128 keys per tile (two blocks of 64, or one of 128).
//      A row whose own tile selected the block weights it exactly; a row whose
//      tile did not gives the block its virtual-token weight alpha on every
//      token (from the mean of that block's logits, which is q . kbar_j), so
//      the PV product yields alpha vsum_j;
//   2. virtual tiles: 128 centroids kbar_j (bf16) as keys and value sums
//      vsum_j (bf16) as values; a column gets alpha_tj unless its block is in
//      the CTA's union (already counted in step 1) or past nblk;
//   3. epilogue: G = Q H-bar^T on the tensor cores into the freed S columns,
//      o_t = (O_t + A_t G_t) / D_t with A_t = sum_{j in U_i} alpha_tj.
// Pipeline, TMEM plan, warp roles, lazy running max, bounded waits and the
// hand-over of P in two halves of 64 keys are those of the token-form kernel
// (attn_tc.cuh).
#pragma once

#include <cudaTypedefs.h>

#include <string>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace pisa {

template <int D, int BS>
struct HybCfg {
    static constexpr int NK = 128;
    static constexpr int MQ = 128;
    static constexpr int NS = (D == 128) ? 2 : 4;
    static constexpr int NBOX = D / 64;
    static constexpr uint32_t BOX_BYTES = 128 * 128;  // 128 rows x 128 bytes
    static constexpr uint32_t TILE_BYTES = NBOX * BOX_BYTES;
    static constexpr uint32_t HALF_BYTES = 64 * 128;  // one 64-row box
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t K_OFF = Q_OFF + 2 * TILE_BYTES;
    static constexpr uint32_t V_OFF = K_OFF + NS * TILE_BYTES;
    static constexpr uint32_t BAR_OFF = V_OFF + NS * TILE_BYTES;
    static constexpr uint32_t NBAR = 1 + 4 * NS + 2 + 2 + 2 + 2 + 1 + 1;
    static constexpr uint32_t SCHED_OFF = BAR_OFF + NBAR * 8 + 16;
    static constexpr int NQT = 256 / BS;  // query tiles per CTA
    static constexpr int MAXBLK = 4096;   // schedule capacity (nblk limit of the library)
    // schedule: union words [128] u32, query-tile mask words [NQT][128] u32, block list [MAXBLK] u16
    static constexpr uint32_t SCHED_BYTES = 4 * 128 + 4 * NQT * 128 + 2 * MAXBLK;
    static constexpr uint32_t SMEM = SCHED_OFF + SCHED_BYTES + 1024;
    static constexpr uint32_t O_COL0 = 256;
    static constexpr uint32_t TMEM_COLS = 512;
};

template <int D, int BS, int ORDER>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_hybrid_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kb,
                       const __grid_constant__ CUtensorMap tm_vs, const __grid_constant__ CUtensorMap tm_hb,
                       const uint32_t* __restrict__ mask, bf16* __restrict__ out, int L, int nblk, int words,
                       const float* __restrict__ wmat, unsigned* status) {
    // ORDER: 0 zeroth, 1 first (H-bar), 3 first + the pooled diagonal second-order
    // term of wmat ([BH, nblk, nblk], row = query tile, gated) on every virtual token
    using C = HybCfg<D, BS>;
    // two K/V stages: stages are freed off group 1's S-full barrier (see the
    // token-form kernel), with no empty-barrier commits in the MMA stream
    constexpr bool kSfullRelease = (C::NS == 2);
    constexpr float LOG2E = 1.4426950408889634f;
    constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, false);
    constexpr uint32_t IDESC_O = tc::idesc_bf16(128, D, true);
    constexpr uint32_t IDESC_G = tc::idesc_bf16(128, D, false);  // G = Q H-bar^T, N = d

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_addr(smem);
    uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + C::NBAR * 8);
    uint32_t* uwords = (uint32_t*)(smem + C::SCHED_OFF);         // [128] union of the CTA's selections
    uint32_t* qwords = uwords + 128;                              // [NQT][128] per query tile
    uint16_t* blist = (uint16_t*)(qwords + C::NQT * 128);         // [MAXBLK] union blocks ascending
    auto bar = [&](int i) { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
    const int B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 1 + C::NS, B_VFULL = 1 + 2 * C::NS, B_VEMPTY = 1 + 3 * C::NS;
    const int B_SFULL = 1 + 4 * C::NS, B_PHALF = B_SFULL + 2, B_PFULL = B_PHALF + 2, B_OFULL = B_PFULL + 2;
    const int B_DONE = B_OFULL + 2, B_HFULL = B_DONE + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = blockIdx.y;
    const int q0 = blockIdx.x * 256;
    const int qt0 = q0 / BS;
    bool aborted = false;

    // ---- schedule: per-tile selection words, their union, the union block list
    for (int e = threadIdx.x; e < C::NQT * words; e += kTcThreads) {
        const int t = e / words, w = e % words;
        const int qt = min(qt0 + t, nblk - 1);
        qwords[t * 128 + w] = __ldg(mask + ((size_t)bh * nblk + qt) * words + w);
    }
    __syncthreads();
    for (int w = threadIdx.x; w < words; w += kTcThreads) {
        uint32_t u = 0u;
        for (int t = 0; t < C::NQT; ++t) u |= qwords[t * 128 + w];
        uwords[w] = u;
    }
    __syncthreads();
    if (warp == 0) {
        int base = 0;
        for (int w0 = 0; w0 < words; w0 += 32) {
            const int w = w0 + lane;
            const uint32_t u = w < words ? uwords[w] : 0u;
            const int cnt = __popc(u);
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            int pos = base + incl - cnt;
            uint32_t b = u;
            while (b) {
                const int x = __ffs(b) - 1;
                blist[pos++] = (uint16_t)(w * 32 + x);
                b &= b - 1;
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) tmem_slot[1] = (uint32_t)base;  // union size
    }
    __syncthreads();
    const int nu = (int)tmem_slot[1];
    constexpr int BPT = C::NK / BS;
    const int nut = (nu + BPT - 1) / BPT;   // union tiles
    const int nvt = (nblk + 127) / 128;     // virtual tiles
    const int NT = nut + nvt;

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
        tc::mbar_init(bar(B_HFULL), 1);
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
            tc::tma_prefetch(&tm_kb);
            tc::tma_prefetch(&tm_vs);
            const int row0 = bh * L + q0;
            tc::mbar_expect_tx(bar(B_QFULL), 2 * C::TILE_BYTES);
            for (int h = 0; h < 2; ++h)
                for (int b = 0; b < C::NBOX; ++b)
                    tc::tma_load_2d(sbase + C::Q_OFF + h * C::TILE_BYTES + b * C::BOX_BYTES, &tm_q, bar(B_QFULL),
                                    b * 64, row0 + h * C::MQ);
            auto load_tile = [&](int jt, uint32_t kdst, uint32_t vdst, bool is_k) {
                const uint32_t br = bar(is_k ? B_KFULL + jt % C::NS : B_VFULL + jt % C::NS);
                tc::mbar_expect_tx(br, C::TILE_BYTES);
                if (jt < nut) {
                    // union tile: BPT blocks of BS rows (a missing second block repeats the first; weight 0)
                    for (int b = 0; b < BPT; ++b) {
                        const int li = jt * BPT + b;
                        const int blk = blist[li < nu ? li : nu - 1];
                        for (int x = 0; x < C::NBOX; ++x)
                            tc::tma_load_2d((is_k ? kdst : vdst) + x * C::BOX_BYTES + b * (BS * 128),
                                            is_k ? &tm_k : &tm_v, br, x * 64, bh * L + blk * BS);
                    }
                } else {
                    const int vt = jt - nut;
                    for (int x = 0; x < C::NBOX; ++x)
                        tc::tma_load_2d((is_k ? kdst : vdst) + x * C::BOX_BYTES, is_k ? &tm_kb : &tm_vs, br, x * 64,
                                        bh * nblk + vt * 128);
                }
            };
            for (int jt = 0; jt < NT; ++jt) {
                const int st = jt % C::NS, u = jt / C::NS;
                if (kSfullRelease) {
                    // S1(jt-1) done: the stage of tile jt-2 is free (one wait per tile, in order)
                    if (jt >= 1 && !tc::mbar_wait(bar(B_SFULL + 1), (jt - 1) & 1, aborted, status, kWaitLimitCycles))
                        break;
                } else if (u > 0 &&
                           !tc::mbar_wait(bar(B_KEMPTY + st), (u - 1) & 1, aborted, status, kWaitLimitCycles)) {
                    break;
                }
                load_tile(jt, sbase + C::K_OFF + st * C::TILE_BYTES, 0, true);
                if (!kSfullRelease && u > 0 &&
                    !tc::mbar_wait(bar(B_VEMPTY + st), (u - 1) & 1, aborted, status, kWaitLimitCycles))
                    break;
                load_tile(jt, 0, sbase + C::V_OFF + st * C::TILE_BYTES, false);
            }
            if (ORDER >= 1 && !aborted) {
                // H-bar into the next K stage once it is free
                const int st = NT % C::NS, u = NT / C::NS;
                const bool free_stage =
                    kSfullRelease ? tc::mbar_wait(bar(B_SFULL + 1), (NT - 1) & 1, aborted, status, kWaitLimitCycles)
                                  : (u == 0 ||
                                     tc::mbar_wait(bar(B_KEMPTY + st), (u - 1) & 1, aborted, status, kWaitLimitCycles));
                if (free_stage) {
                    tc::mbar_expect_tx(bar(B_HFULL), (uint32_t)(D * D * 2));
                    for (int x = 0; x < C::NBOX; ++x)
                        tc::tma_load_2d(sbase + C::K_OFF + st * C::TILE_BYTES + x * C::BOX_BYTES, &tm_hb,
                                        bar(B_HFULL), x * 64, bh * D);
                }
            }
            if (aborted) {
                // give in-flight copies time to land before the CTA exits
                bool a2 = false;
                tc::mbar_wait(bar(B_QFULL), 0, a2, status, kWaitLimitCycles);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint64_t qdesc0 = tc::sdesc_sw128(sbase + C::Q_OFF, 16, 1024);
            const uint64_t kdesc0 = tc::sdesc_sw128(sbase + C::K_OFF, 16, 1024);
            const uint64_t vdesc0 = tc::sdesc_sw128(sbase + C::V_OFF, C::BOX_BYTES, 1024);
            constexpr uint64_t kTileStep = C::TILE_BYTES >> 4;
            auto issue_s = [&](int h, int st, uint32_t idesc) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
                    tc::mma_ss(tmem + (uint32_t)(h * 128), qdesc0 + h * kTileStep + off, kdesc0 + st * kTileStep + off,
                               idesc, kk > 0);
                }
            };
            auto issue_pv = [&](int h, int st, int half, bool first) {
#pragma unroll
                for (int kk = half * 4; kk < half * 4 + 4; ++kk)
                    tc::mma_ts(tmem + C::O_COL0 + h * D, tmem + (uint32_t)(h * 128) + kk * 8,
                               vdesc0 + st * kTileStep + (uint64_t)((kk * 16 * 128) >> 4), IDESC_O,
                               (first && kk == 0) ? 0u : 1u);
            };
            bool ok = tc::mbar_wait(bar(B_QFULL), 0, aborted, status, kWaitLimitCycles);
            ok = ok && tc::mbar_wait(bar(B_KFULL + 0), 0, aborted, status, kWaitLimitCycles);
            if (ok) {
                issue_s(0, 0, IDESC_S);
                tc::mma_commit(bar(B_SFULL + 0));
                issue_s(1, 0, IDESC_S);
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
                if (more) {
                    if (!tc::mbar_wait(bar(B_KFULL + st1), u1 & 1, aborted, status, kWaitLimitCycles)) break;
                    issue_s(0, st1, IDESC_S);
                    tc::mma_commit(bar(B_SFULL + 0));
                }
                if (!tc::mbar_wait(bar(B_PHALF + 1), jt & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                issue_pv(1, st, 0, jt == 0);
                if (!tc::mbar_wait(bar(B_PFULL + 1), jt & 1, aborted, status, kWaitLimitCycles)) break;
                tc::fence_after_sync();
                issue_pv(1, st, 1, false);
                if (!kSfullRelease) tc::mma_commit(bar(B_VEMPTY + st));
                if (more) {
                    issue_s(1, st1, IDESC_S);
                    tc::mma_commit(bar(B_SFULL + 1));
                    if (!kSfullRelease) tc::mma_commit(bar(B_KEMPTY + st1));
                }
            }
            if (!aborted) {
                if (ORDER >= 1) {
                    // G_h = Q_h H-bar^T into the S columns (their P was consumed by the last PV)
                    if (tc::mbar_wait(bar(B_HFULL), 0, aborted, status, kWaitLimitCycles)) {
                        issue_s(0, NT % C::NS, IDESC_G);
                        issue_s(1, NT % C::NS, IDESC_G);
                    }
                }
                tc::mma_commit(bar(B_OFULL + 0));
                tc::mma_commit(bar(B_OFULL + 1));
            }
            tc::mma_commit(bar(B_DONE));
            bool a2 = false;
            tc::mbar_wait(bar(B_DONE), 0, a2, status, kWaitLimitCycles);
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int h = (warp - 2) / 4;
        const int quarter = warp % 4;
        const int r = quarter * 32 + lane;
        const int qrow = q0 + h * C::MQ + r;
        const bool valid = qrow < L;
        const int tq = (h * C::MQ + r) / BS;  // query tile of this row inside the CTA (0 .. NQT-1)
        const uint32_t* myw = qwords + tq * 128;
        const float* wrow = (ORDER == 3) ? wmat + ((size_t)bh * nblk + min(qt0 + tq, nblk - 1)) * nblk : nullptr;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t s_addr = lane_base + (uint32_t)(h * 128);
        const uint32_t o_addr = lane_base + C::O_COL0 + h * D;
        constexpr int CPB = BS / 32;
        const float inv_bs = 1.0f / (float)BS;
        float m_run = -INFINITY;  // running max (log2 units)
        float dsum = 0.f;         // denominator
        float amass = 0.f;        // sum over unselected blocks of alpha (first-order mass)

        for (int jt = 0; jt < NT; ++jt) {
            if (!tc::mbar_wait_warp(bar(B_SFULL + h), jt & 1, aborted, status, kWaitLimitCycles)) break;
            tc::fence_after_sync();
            // the whole 128-column S tile in registers: one TMEM round trip
            uint32_t sv[C::NK];
#pragma unroll
            for (int c = 0; c < C::NK / 32; ++c)
                tc::tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32 * c));
            tc::tmem_wait_ld();
            // per-column weight rule of this tile: 0 = off, 1 = exact e^{x}, 2 = virtual weight
            float mc = -INFINITY;
            bool sel[BPT], live[BPT];
            float l2[BPT];
            uint32_t okw[4] = {0u, 0u, 0u, 0u};
            const bool is_union = jt < nut;
            if (is_union) {
#pragma unroll
                for (int b = 0; b < BPT; ++b) {
                    const int li = jt * BPT + b;
                    live[b] = li < nu;
                    const int blk = blist[live[b] ? li : 0];
                    sel[b] = live[b] && ((myw[blk >> 5] >> (blk & 31)) & 1u);
                    l2[b] = 0.f;
                    if (!live[b]) continue;
                    const uint32_t* x = sv + b * BS;
                    if (sel[b]) {
                        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                        for (int e = 0; e < BS; ++e) m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(x[e]));
                        mc = fmaxf(mc, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * LOG2E);
                    } else {
                        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int e = 0; e < BS; ++e) s4[e & 3] += __uint_as_float(x[e]);
                        float wv = 0.f;
                        if (ORDER == 3) wv = __ldg(wrow + blk);
                        l2[b] = (((s4[0] + s4[1]) + (s4[2] + s4[3])) * inv_bs + wv) * LOG2E;
                        mc = fmaxf(mc, l2[b]);
                    }
                }
            } else {
                // virtual tile: 128 centroids; a column counts unless its block is
                // in the union or past nblk
                const int vj0 = (jt - nut) * 128;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int j = vj0 + 32 * w;
                    uint32_t inb = 0u;
                    if (j < nblk) inb = (nblk - j >= 32) ? 0xffffffffu : ((1u << (nblk - j)) - 1u);
                    okw[w] = inb & ~((j >> 5) < words ? uwords[j >> 5] : 0u);
                }
                if (ORDER == 3) {
                    // the virtual token's logit carries the tile's pooled w (in place)
#pragma unroll
                    for (int e = 0; e < C::NK; ++e)
                        if ((okw[e >> 5] >> (e & 31)) & 1u)
                            sv[e] = __float_as_uint(__uint_as_float(sv[e]) + __ldg(wrow + vj0 + e));
                }
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int e = 0; e < C::NK; ++e) {
                    const float x = ((okw[e >> 5] >> (e & 31)) & 1u) ? __uint_as_float(sv[e]) : -INFINITY;
                    m4[e & 3] = fmaxf(m4[e & 3], x);
                }
                mc = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * LOG2E;
            }
            const bool raise = mc > m_run + 8.0f;
            const float scale = raise ? tc::ex2(m_run - mc) : 1.0f;
            if (raise) {
                dsum *= scale;
                amass *= scale;
                m_run = mc;
            }
            if (__any_sync(0xffffffffu, raise) && jt > 0) {
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
            if (is_union) {
#pragma unroll
                for (int b = 0; b < BPT; ++b) {
                    const uint32_t* x = sv + b * BS;
                    if (live[b] && sel[b]) {
                        float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int c = 0; c < CPB; ++c) {
                            uint32_t pk[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const float xa = __uint_as_float(x[32 * c + 2 * e]);
                                const float xb = __uint_as_float(x[32 * c + 2 * e + 1]);
                                const float a0 = tc::ex2(fmaf(xa, LOG2E, -m_run));
                                const float a1 = (e & 1) ? tc::ex2_fma(fmaf(xb, LOG2E, -m_run))
                                                         : tc::ex2(fmaf(xb, LOG2E, -m_run));
                                d4[e & 3] += a0 + a1;
                                pk[e] = tc::pack_bf16x2(a0, a1);
                            }
                            tc::tmem_st16(s_addr + (b * CPB + c) * 16, pk);
                            if (b * CPB + c == 1) {  // keys 0..63 are in TMEM: hand over the first half
                                tc::tmem_wait_st();
                                tc::fence_before_sync();
                                tc::mbar_arrive(bar(B_PHALF + h));
                            }
                        }
                        dsum += (d4[0] + d4[1]) + (d4[2] + d4[3]);
                    } else {
                        // unselected (virtual-token weight on every token) or padding (weight 0)
                        const float alpha = live[b] ? tc::ex2(l2[b] - m_run) : 0.f;
                        dsum = fmaf((float)BS, alpha, dsum);
                        amass += alpha;
                        uint32_t pk[16];
                        const uint32_t a2 = tc::pack_bf16x2(alpha, alpha);
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = a2;
#pragma unroll
                        for (int c = 0; c < CPB; ++c) {
                            tc::tmem_st16(s_addr + (b * CPB + c) * 16, pk);
                            if (b * CPB + c == 1) {
                                tc::tmem_wait_st();
                                tc::fence_before_sync();
                                tc::mbar_arrive(bar(B_PHALF + h));
                            }
                        }
                    }
                }
            } else {
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int e0 = 32 * c + 2 * e;
                        const float a0 = ((okw[c] >> (2 * e)) & 1u) ? tc::ex2(fmaf(__uint_as_float(sv[e0]), LOG2E, -m_run))
                                                                    : 0.f;
                        // a quarter of the exponentials on the FMA pipe, as in the union tiles
                        const float x1 = fmaf(__uint_as_float(sv[e0 + 1]), LOG2E, -m_run);
                        const float a1 = ((okw[c] >> (2 * e + 1)) & 1u) ? ((e & 1) ? tc::ex2_fma(x1) : tc::ex2(x1))
                                                                        : 0.f;
                        a4[e & 3] += a0 + a1;
                        pk[e] = tc::pack_bf16x2(a0, a1);
                    }
                    tc::tmem_st16(s_addr + c * 16, pk);
                    if (c == 1) {
                        tc::tmem_wait_st();
                        tc::fence_before_sync();
                        tc::mbar_arrive(bar(B_PHALF + h));
                    }
                }
                const float asum = (a4[0] + a4[1]) + (a4[2] + a4[3]);
                dsum = fmaf((float)BS, asum, dsum);
                amass += asum;
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_PFULL + h));
        }
        // epilogue: o = (O + A G) / D, G = H-bar q in the S columns
        if (tc::mbar_wait_warp(bar(B_OFULL + h), 0, aborted, status, kWaitLimitCycles)) {
            tc::fence_after_sync();
            const float inv = 1.0f / dsum;
            bf16* orow = out + ((size_t)bh * L + (valid ? qrow : 0)) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t raw[32], g[32];
                tc::tmem_ld32(o_addr + c * 32, raw);
                if (ORDER >= 1) tc::tmem_ld32(s_addr + c * 32, g);
                tc::tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float x0 = __uint_as_float(raw[2 * e]), x1 = __uint_as_float(raw[2 * e + 1]);
                    if (ORDER >= 1) {
                        x0 = fmaf(amass, __uint_as_float(g[2 * e]), x0);
                        x1 = fmaf(amass, __uint_as_float(g[2 * e + 1]), x1);
                    }
                    pk[e] = tc::pack_bf16x2(x0 * inv, x1 * inv);
                }
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

// Host: tensor maps and launch of the hybrid kernel.  kbar_bf, vsum_bf: [BH, nblk, d] bf16;
// hbar_bf: [BH, d, d] bf16 (row = value channel).  Requires L % 128 == 0 (checked by the caller).
// order 3 = first order + the pooled w matrix `wmat` (the hybrid's second order).
inline pisa_status run_attn_hybrid(const void* q, const void* k, const void* v, const void* kbar_bf,
                                   const void* vsum_bf, const void* hbar_bf, const uint32_t* mask, void* out,
                                   long BH, int L, int d, int B, int nblk, int words, int order, const float* wmat,
                                   unsigned* status, cudaStream_t s, std::string* err) {
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
    auto make = [&](CUtensorMap* m, const void* p, long rows, int box_rows) -> bool {
        cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)rows};
        cuuint64_t gstride[1] = {(cuuint64_t)d * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
        cuuint32_t estride[2] = {1, 1};
        return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p), gdim, gstride, box, estride,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    CUtensorMap mq, mk, mv, mkb, mvs, mhb;
    if (!make(&mq, q, BH * L, 128) || !make(&mk, k, BH * L, B) || !make(&mv, v, BH * L, B) ||
        !make(&mkb, kbar_bf, BH * nblk, 128) || !make(&mvs, vsum_bf, BH * nblk, 128) ||
        !make(&mhb, hbar_bf, BH * d, d)) {
        *err = "cuTensorMapEncodeTiled failed for the hybrid kernel";
        return PISA_ERR_CUDA;
    }
    dim3 grid((unsigned)((L + 255) / 256), (unsigned)BH);
    cudaError_t e = cudaSuccess;
#define PISA_HYB_LAUNCH(DD, BB, OO)                                                                             \
    if (d == DD && B == BB && order == OO) {                                                                    \
        auto kern = attn_hybrid_kernel<DD, BB, OO>;                                                             \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)HybCfg<DD, BB>::SMEM); \
        if (e == cudaSuccess) {                                                                                 \
            kern<<<grid, kTcThreads, HybCfg<DD, BB>::SMEM, s>>>(mq, mk, mv, mkb, mvs, mhb, mask, (bf16*)out, L,   \
                                                                nblk, words, wmat, status);                     \
            e = cudaGetLastError();                                                                             \
        }                                                                                                       \
    } else
    PISA_HYB_LAUNCH(64, 64, 0)
    PISA_HYB_LAUNCH(64, 64, 1)
    PISA_HYB_LAUNCH(64, 64, 3)
    PISA_HYB_LAUNCH(64, 128, 0)
    PISA_HYB_LAUNCH(64, 128, 1)
    PISA_HYB_LAUNCH(64, 128, 3)
    PISA_HYB_LAUNCH(128, 64, 0)
    PISA_HYB_LAUNCH(128, 64, 1)
    PISA_HYB_LAUNCH(128, 64, 3)
    PISA_HYB_LAUNCH(128, 128, 0)
    PISA_HYB_LAUNCH(128, 128, 1)
    PISA_HYB_LAUNCH(128, 128, 3) {
        *err = "no hybrid kernel for this d/B/order";
        return PISA_ERR_UNSUPPORTED;
    }
#undef PISA_HYB_LAUNCH
    if (e != cudaSuccess) {
        *err = std::string("attn_hybrid_kernel launch: ") + cudaGetErrorString(e);
        return PISA_ERR_CUDA;
    }
    return PISA_OK;
}

}  // namespace pisa
