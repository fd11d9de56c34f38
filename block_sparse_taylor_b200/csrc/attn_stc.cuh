// Piecewise sparse attention on tcgen05 tensor cores, statistics form: the
// first-order term of an unselected block is the contraction H_j q_t with the
// block's d x d statistic (the FLOP-minimal association when d <= B).
//
// What it computes (PISA paper, section 3.2 "Formulation" and "Practical
// Challenge"; "Sparse Linear Attention" blog, section "Sparse Linear
// Attention"; the pooled second order of the blog's PWT section): for query
// row t of tile i,
//   D_t = sum_{j in S_i} sum_n e^{q.k_n} + sum_{j in U_i} B e^{l_tj}
//   N_t = sum_{j in S_i} sum_n e^{q.k_n} v_n + sum_{j in U_i} e^{l_tj} (vsum_j + H_j q_t)
//   o_t = N_t / D_t,  l_tj = q_t.kbar_j (+ the pooled w_ij for ORDER 3).
//
// One CTA = 256 query rows of one (batch, head) = two 128-row M tiles, in two
// phases that share one running max and one denominator per row:
//   phase 1, the union tiles: the blocks selected by any query tile of the CTA,
//     ascending, 128 keys per tile, through S = Q K^T and O += P V exactly as in
//     the token-form kernel: a row whose own tile selected the block weights its
//     keys e^{x}; any other row gives them the first-order token weights
//     e^{l}(1 + x_n - s-bar), whose PV sum is e^{l}(vsum_j + H_j q_t), so these
//     blocks are counted once, and correctly, for every row;
//   phase 2, every other block (unselected by all of the CTA's tiles): one MMA
//     per M tile and item of GB blocks, G = Q [H_j ; kbar_j]^T with N = GB d + 16:
//     the first GB d columns are H_j q_t, and two more columns per block hold
//     q_t . kbar_j as the sum of a bf16 high part and a bf16 low part of the fp32
//     centroid (the "aug" rows of the statistics).  The softmax warps read G back
//     from TMEM and accumulate e^{l - m}(G + vsum_j) in registers, so the row
//     weight is applied on the way out and the tensor core never waits for it;
//     vsum_j comes through a ring of shared-memory slots that the producer fills
//     with bulk copies, so the softmax reads it at shared-memory latency.
// The phase-1 accumulator O is read into the same registers between the phases.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator and MMA issuer, warps
// 2-3 idle (warpgroup 0 runs on 120 registers a thread: the MMA issuer keeps
// its operand descriptors in registers), warps 4-7 and 8-11 the softmax groups
// of M tiles 0 and 1 (192 registers a thread: the phase-2 accumulator alone
// takes d of them; with one budget of 168 for all threads the d = 128 variants
// spilled it).  The split uses exactly the registers the CTA is launched with,
// 384 x 168 = 128 x 120 + 256 x 192, and the host checks that count before
// each launch.  TMEM ping-pong of phase 1, bounded
// waits and the lazy running max (raised only when it grows by more than 2^8)
// are those of the token-form kernel (attn_tc.cuh).  TMEM: phase 1 S0 | S1 | O0 | O1; phase 2 three G slots
// of 144 columns at columns 0, 160 and 320, used by the items in turn (M tile 0
// and M tile 1 of each item), so the MMA runs up to two slots ahead.
#pragma once

#include <cudaTypedefs.h>

#include <string>

#include "attn_tc.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace pisa {

// Threads of the statistics-form kernel and its register split (see above).
constexpr int kStcThreads = 384;
constexpr uint32_t kStcRegsLaunch = 168;  // per thread at launch (65536 / 384, in steps of 8)
constexpr uint32_t kStcRegsSupport = 120;  // warpgroup 0: producer, MMA, two idle warps
constexpr uint32_t kStcRegsSoftmax = 192;  // warpgroups 1 and 2
static_assert(128 * kStcRegsSupport + 256 * kStcRegsSoftmax <= kStcThreads * kStcRegsLaunch,
              "register split exceeds the launch allocation");

template <int D, int BS>
struct StcCfg {
    static constexpr int NK = 128;                 // keys per union tile
    static constexpr int MQ = 128;                 // rows per M tile
    static constexpr int NS = (D == 128) ? 2 : 4;  // phase-1 K/V stages
    static constexpr int NBOX = D / 64;            // 64-column (128-byte) swizzle boxes per row
    static constexpr uint32_t BOX_BYTES = 128 * 128;
    static constexpr uint32_t TILE_BYTES = NBOX * BOX_BYTES;
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t KV_OFF = Q_OFF + 2 * TILE_BYTES;
    static constexpr uint32_t K_OFF = KV_OFF;
    static constexpr uint32_t V_OFF = K_OFF + NS * TILE_BYTES;
    static constexpr uint32_t KV_BYTES = 2 * NS * TILE_BYTES;
    // phase 2: an item is GB key blocks; its B operand is GB H_j (D rows each)
    // followed by 16 rows for the centroids (8 per block: high, low, zeros)
    static constexpr int GB = (D == 64) ? 2 : 1;
    static constexpr int N2 = GB * D + 16;               // 144 in both cases
    static constexpr uint32_t AUG_ROW0 = GB * D;         // first centroid row (and G column)
    static constexpr uint32_t BOX2_BYTES = N2 * 128;     // one 64-column box of a stage
    static constexpr uint32_t STAGE2_BYTES = NBOX * BOX2_BYTES;
    static constexpr uint32_t STAGE2_TX = GB * (D * D * 2 + 8 * D * 2);  // bytes a stage load brings
    static constexpr int NS2 = (KV_BYTES / STAGE2_BYTES) < 4 ? (int)(KV_BYTES / STAGE2_BYTES) : 4;
    static constexpr int NSLOT = 3;
    static constexpr uint32_t SLOT_STRIDE = 160;         // TMEM columns between G slots
    static constexpr int NQT = 256 / BS;                 // query tiles per CTA
    static constexpr int MAXBLK = 4096;                  // nblk limit of the library
    // phase 2: the items' value sums (fp32, GB blocks each) through their own ring of
    // NV slots, filled by bulk copies and released by the softmax threads
    static constexpr int NV = 4;
    static constexpr uint32_t VS_BYTES = GB * D * 4;
    static constexpr uint32_t VS_OFF = KV_OFF + KV_BYTES;
    // QFULL; KFULL, KEMPTY, VFULL, VEMPTY per stage; SFULL, PHALF, PFULL, OFULL per
    // M tile; ODRAIN; F2FULL, F2EMPTY per phase-2 stage; GFULL, GEMPTY per slot; DONE;
    // VSFULL, VSEMPTY per value-sum slot
    static constexpr uint32_t NBAR = 1 + 4 * NS + 8 + 1 + 2 * NS2 + 2 * NSLOT + 1 + 2 * NV;
    static constexpr uint32_t BAR_OFF = VS_OFF + NV * VS_BYTES;
    static constexpr uint32_t SCHED_OFF = BAR_OFF + NBAR * 8 + 16;
    // schedule: union words [128], per-tile words [NQT][128], union list [MAXBLK],
    // list of the other blocks [MAXBLK]
    static constexpr uint32_t SCHED_BYTES = 4 * 128 + 4 * NQT * 128 + 2 * MAXBLK * 2;
    static constexpr uint32_t SMEM = SCHED_OFF + SCHED_BYTES + 1024;
    static constexpr uint32_t O_COL0 = 256;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(NS2 >= 2, "phase 2 needs two stages");
    static_assert(STAGE2_BYTES % 1024 == 0 && BOX2_BYTES % 1024 == 0, "swizzle atoms need 1024-byte bases");
    static_assert((NSLOT - 1) * SLOT_STRIDE + N2 <= TMEM_COLS, "G slots exceed TMEM");
    static_assert(O_COL0 + 2 * D <= TMEM_COLS, "O exceeds TMEM");
};

template <int D, int BS, int ORDER>
__global__ void __launch_bounds__(kStcThreads, 1)
    attn_stc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_h,
                    const __grid_constant__ CUtensorMap tm_aug, const uint32_t* __restrict__ mask,
                    const float* __restrict__ vsum, bf16* __restrict__ out, int L, int nblk, int words, int gate,
                    float ln_b, const float* __restrict__ wmat, unsigned* status, float* __restrict__ lse) {
    // ORDER: 1 first order; 3 first order + the pooled diagonal w of wmat
    // ([BH, nblk, nblk], row = query tile, already gated) on every unselected block
    static_assert(ORDER == 1 || ORDER == 3, "statistics-form kernel: orders 1 and 3");
    using C = StcCfg<D, BS>;
    constexpr bool kSfullRelease = (C::NS == 2);
    constexpr float LOG2E = 1.4426950408889634f;
    constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, false);  // S = Q K^T
    constexpr uint32_t IDESC_O = tc::idesc_bf16(128, D, true);     // O += P V
    constexpr uint32_t IDESC_G = tc::idesc_bf16(128, C::N2, false);  // G = Q [H ; kbar]^T

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_addr(smem);
    uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + C::NBAR * 8);
    uint32_t* uwords = (uint32_t*)(smem + C::SCHED_OFF);   // [128] union of the CTA's selections
    uint32_t* qwords = uwords + 128;                        // [NQT][128] per query tile
    uint16_t* blist = (uint16_t*)(qwords + C::NQT * 128);   // [MAXBLK] union blocks, ascending
    uint16_t* nlist = blist + C::MAXBLK;                    // [MAXBLK] the other blocks, ascending
    auto bar = [&](int i) { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
    const int B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 1 + C::NS, B_VFULL = 1 + 2 * C::NS, B_VEMPTY = 1 + 3 * C::NS;
    const int B_SFULL = 1 + 4 * C::NS, B_PHALF = B_SFULL + 2, B_PFULL = B_PHALF + 2, B_OFULL = B_PFULL + 2;
    const int B_ODRAIN = B_OFULL + 2, B_F2FULL = B_ODRAIN + 1, B_F2EMPTY = B_F2FULL + C::NS2;
    const int B_GFULL = B_F2EMPTY + C::NS2, B_GEMPTY = B_GFULL + C::NSLOT, B_DONE = B_GEMPTY + C::NSLOT;
    const int B_VSFULL = B_DONE + 1, B_VSEMPTY = B_VSFULL + C::NV;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = blockIdx.y;
    const int q0 = blockIdx.x * 256;
    const int qt0 = q0 / BS;
    bool aborted = false;

    // ---- schedule: per-tile selection words, their union, the union list and the rest
    for (int e = threadIdx.x; e < C::NQT * words; e += kStcThreads) {
        const int t = e / words, w = e % words;
        const int qt = min(qt0 + t, nblk - 1);
        qwords[t * 128 + w] = __ldg(mask + ((size_t)bh * nblk + qt) * words + w);
    }
    __syncthreads();
    for (int w = threadIdx.x; w < words; w += kStcThreads) {
        uint32_t u = 0u;
        for (int t = 0; t < C::NQT; ++t) u |= qwords[t * 128 + w];
        uwords[w] = u;
    }
    __syncthreads();
    if (warp == 0) {
        int base_u = 0, base_n = 0;
        for (int w0 = 0; w0 < words; w0 += 32) {
            const int w = w0 + lane;
            uint32_t inb = 0u;
            if (w < words) inb = (nblk - 32 * w >= 32) ? 0xffffffffu : ((1u << (nblk - 32 * w)) - 1u);
            const uint32_t u = w < words ? uwords[w] : 0u;
            const uint32_t n = inb & ~u;
            const int cu = __popc(u), cn = __popc(n);
            int iu = cu, in = cn;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int vu = __shfl_up_sync(0xffffffffu, iu, o);
                const int vn = __shfl_up_sync(0xffffffffu, in, o);
                if (lane >= o) {
                    iu += vu;
                    in += vn;
                }
            }
            int pu = base_u + iu - cu, pn = base_n + in - cn;
            for (uint32_t b = u; b; b &= b - 1) blist[pu++] = (uint16_t)(w * 32 + __ffs(b) - 1);
            for (uint32_t b = n; b; b &= b - 1) nlist[pn++] = (uint16_t)(w * 32 + __ffs(b) - 1);
            base_u += __shfl_sync(0xffffffffu, iu, 31);
            base_n += __shfl_sync(0xffffffffu, in, 31);
        }
        if (lane == 0) {
            tmem_slot[1] = (uint32_t)base_u;
            tmem_slot[2] = (uint32_t)base_n;
        }
    }
    __syncthreads();
    const int nu = (int)tmem_slot[1];     // union blocks
    const int nn = (int)tmem_slot[2];     // the other blocks (nu + nn == nblk)
    constexpr int BPT = C::NK / BS;       // blocks per union tile
    const int NT = (nu + BPT - 1) / BPT;  // union tiles (phase 1)
    const int NI = (nn + C::GB - 1) / C::GB;  // items (phase 2)

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
        tc::mbar_init(bar(B_ODRAIN), 256);
        for (int s = 0; s < C::NS2; ++s) {
            tc::mbar_init(bar(B_F2FULL + s), 1);
            tc::mbar_init(bar(B_F2EMPTY + s), 1);
        }
        for (int s = 0; s < C::NSLOT; ++s) {
            tc::mbar_init(bar(B_GFULL + s), 1);
            tc::mbar_init(bar(B_GEMPTY + s), 128);
        }
        tc::mbar_init(bar(B_DONE), 1);
        for (int s = 0; s < C::NV; ++s) {
            tc::mbar_init(bar(B_VSFULL + s), 1);
            tc::mbar_init(bar(B_VSEMPTY + s), 256);
        }
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

    if (warp < 4) {
      tc::reg_dealloc<kStcRegsSupport>();
      if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tc::tma_prefetch(&tm_q);
            tc::tma_prefetch(&tm_k);
            tc::tma_prefetch(&tm_v);
            tc::tma_prefetch(&tm_h);
            tc::tma_prefetch(&tm_aug);
            const int row0 = bh * L + q0;
            tc::mbar_expect_tx(bar(B_QFULL), 2 * C::TILE_BYTES);
            for (int h = 0; h < 2; ++h)
                for (int b = 0; b < C::NBOX; ++b)
                    tc::tma_load_2d(sbase + C::Q_OFF + h * C::TILE_BYTES + b * C::BOX_BYTES, &tm_q, bar(B_QFULL),
                                    b * 64, row0 + h * C::MQ);
            // phase 1: union tiles (BPT blocks of BS rows; a missing second block repeats the first)
            auto load_tile = [&](int jt, uint32_t dst, bool is_k) {
                const uint32_t br = bar(is_k ? B_KFULL + jt % C::NS : B_VFULL + jt % C::NS);
                tc::mbar_expect_tx(br, C::TILE_BYTES);
                for (int b = 0; b < BPT; ++b) {
                    const int li = jt * BPT + b;
                    const int blk = blist[li < nu ? li : nu - 1];
                    for (int x = 0; x < C::NBOX; ++x)
                        tc::tma_load_2d(dst + x * C::BOX_BYTES + b * (BS * 128), is_k ? &tm_k : &tm_v, br, x * 64,
                                        bh * L + blk * BS);
                }
            };
            for (int jt = 0; jt < NT; ++jt) {
                const int st = jt % C::NS, u = jt / C::NS;
                if (kSfullRelease) {
                    if (jt >= 1 && !tc::mbar_wait(bar(B_SFULL + 1), (jt - 1) & 1, aborted, status, kWaitLimitCycles))
                        break;
                } else if (u > 0 &&
                           !tc::mbar_wait(bar(B_KEMPTY + st), (u - 1) & 1, aborted, status, kWaitLimitCycles)) {
                    break;
                }
                load_tile(jt, sbase + C::K_OFF + st * C::TILE_BYTES, true);
                if (!kSfullRelease && u > 0 &&
                    !tc::mbar_wait(bar(B_VEMPTY + st), (u - 1) & 1, aborted, status, kWaitLimitCycles))
                    break;
                load_tile(jt, sbase + C::V_OFF + st * C::TILE_BYTES, false);
            }
            // phase 2: the stages overlay the K/V ring, so wait until every phase-1
            // MMA has completed (OFULL of M tile 1 is committed after all of them)
            if (!aborted && NI > 0 && NT > 0) tc::mbar_wait(bar(B_OFULL + 1), 0, aborted, status, kWaitLimitCycles);
            for (int g = 0; !aborted && g < NI; ++g) {
                const int st = g % C::NS2, u = g / C::NS2;
                if (u > 0 && !tc::mbar_wait(bar(B_F2EMPTY + st), (u - 1) & 1, aborted, status, kWaitLimitCycles))
                    break;
                const uint32_t dst = sbase + C::KV_OFF + st * C::STAGE2_BYTES;
                tc::mbar_expect_tx(bar(B_F2FULL + st), C::STAGE2_TX);
                for (int b = 0; b < C::GB; ++b) {
                    const int li = g * C::GB + b;
                    const int blk = nlist[li < nn ? li : nn - 1];
                    const int hrow = (bh * nblk + blk) * D, arow = (bh * nblk + blk) * 8;
                    for (int x = 0; x < C::NBOX; ++x) {
                        tc::tma_load_2d(dst + x * C::BOX2_BYTES + b * (D * 128), &tm_h, bar(B_F2FULL + st), x * 64,
                                        hrow);
                        tc::tma_load_2d(dst + x * C::BOX2_BYTES + C::AUG_ROW0 * 128 + b * 1024, &tm_aug,
                                        bar(B_F2FULL + st), x * 64, arow);
                    }
                }
                // the item's value sums into their slot, once the softmax is done with the slot's last item
                const int vs = g % C::NV, vu = g / C::NV;
                if (vu > 0 && !tc::mbar_wait(bar(B_VSEMPTY + vs), (vu - 1) & 1, aborted, status, kWaitLimitCycles))
                    break;
                tc::mbar_expect_tx(bar(B_VSFULL + vs), C::VS_BYTES);
                for (int b = 0; b < C::GB; ++b) {
                    const int li = g * C::GB + b;
                    const int blk = nlist[li < nn ? li : nn - 1];
                    tc::bulk_load(sbase + C::VS_OFF + vs * C::VS_BYTES + b * D * 4,
                                  vsum + ((size_t)bh * nblk + blk) * D, D * 4, bar(B_VSFULL + vs));
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
            const uint64_t gdesc0 = tc::sdesc_sw128(sbase + C::KV_OFF, 16, 1024);
            constexpr uint64_t kTileStep = C::TILE_BYTES >> 4;
            constexpr uint64_t kStage2Step = C::STAGE2_BYTES >> 4;
            auto issue_s = [&](int h, int st) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
                    tc::mma_ss(tmem + (uint32_t)(h * 128), qdesc0 + h * kTileStep + off, kdesc0 + st * kTileStep + off,
                               IDESC_S, kk > 0);
                }
            };
            auto issue_pv = [&](int h, int st, int half, bool first) {
#pragma unroll
                for (int kk = half * 4; kk < half * 4 + 4; ++kk)
                    tc::mma_ts(tmem + C::O_COL0 + h * D, tmem + (uint32_t)(h * 128) + kk * 8,
                               vdesc0 + st * kTileStep + (uint64_t)((kk * 16 * 128) >> 4), IDESC_O,
                               (first && kk == 0) ? 0u : 1u);
            };
            auto issue_g = [&](int h, int st, uint32_t dcol) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t qoff = ((kk / 4) * C::BOX_BYTES + (kk % 4) * 32) >> 4;
                    const uint64_t goff = ((kk / 4) * C::BOX2_BYTES + (kk % 4) * 32) >> 4;
                    tc::mma_ss(tmem + dcol, qdesc0 + h * kTileStep + qoff, gdesc0 + st * kStage2Step + goff, IDESC_G,
                               kk > 0);
                }
            };
            bool ok = tc::mbar_wait(bar(B_QFULL), 0, aborted, status, kWaitLimitCycles);
            if (ok && NT > 0) {
                ok = tc::mbar_wait(bar(B_KFULL + 0), 0, aborted, status, kWaitLimitCycles);
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
                    if (!kSfullRelease) tc::mma_commit(bar(B_VEMPTY + st));
                    if (more) {
                        issue_s(1, st1);
                        tc::mma_commit(bar(B_SFULL + 1));
                        if (!kSfullRelease) tc::mma_commit(bar(B_KEMPTY + st1));
                    }
                }
                if (!aborted) {
                    tc::mma_commit(bar(B_OFULL + 0));
                    tc::mma_commit(bar(B_OFULL + 1));
                }
                // phase 2 writes over O: both softmax groups must have read it
                if (!aborted && NI > 0) tc::mbar_wait(bar(B_ODRAIN), 0, aborted, status, kWaitLimitCycles);
            }
            for (int g = 0; !aborted && g < NI; ++g) {
                const int st = g % C::NS2, u = g / C::NS2;
                if (!tc::mbar_wait(bar(B_F2FULL + st), u & 1, aborted, status, kWaitLimitCycles)) break;
                for (int h = 0; h < 2; ++h) {
                    const int it = 2 * g + h, slot = it % C::NSLOT, use = it / C::NSLOT;
                    if (use > 0 &&
                        !tc::mbar_wait(bar(B_GEMPTY + slot), (use - 1) & 1, aborted, status, kWaitLimitCycles))
                        break;
                    tc::fence_after_sync();
                    issue_g(h, st, (uint32_t)(slot * C::SLOT_STRIDE));
                    tc::mma_commit(bar(B_GFULL + slot));
                }
                if (aborted) break;
                tc::mma_commit(bar(B_F2EMPTY + st));
            }
            // every MMA issued by this thread has completed before TMEM is freed
            tc::mma_commit(bar(B_DONE));
            bool a2 = false;
            tc::mbar_wait(bar(B_DONE), 0, a2, status, kWaitLimitCycles);
        }
      }
    } else {
        tc::reg_alloc<kStcRegsSoftmax>();
        // ------------------------------------------------------------- softmax
        const int h = (warp - 4) / 4;             // M tile of this group
        const int quarter = warp % 4;             // TMEM lane quarter of this warp
        const int r = quarter * 32 + lane;        // row inside the M tile = TMEM lane
        const int qrow = q0 + h * C::MQ + r;      // query row inside the head
        const bool valid = qrow < L;
        const int tq = (h * C::MQ + r) / BS;      // query tile of this row inside the CTA
        const uint32_t* myw = qwords + tq * 128;
        const float* wrow = (ORDER == 3) ? wmat + ((size_t)bh * nblk + min(qt0 + tq, nblk - 1)) * nblk : nullptr;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t s_addr = lane_base + (uint32_t)(h * 128);
        const uint32_t o_addr = lane_base + C::O_COL0 + h * D;
        float m_run = -INFINITY;  // running max (log2 units)
        float dsum = 0.f;         // denominator (scaled by 2^-m_run)

        // ---- phase 1: union tiles
        for (int jt = 0; jt < NT; ++jt) {
            if (!tc::mbar_wait_warp(bar(B_SFULL + h), jt & 1, aborted, status, kWaitLimitCycles)) break;
            tc::fence_after_sync();
            bool sel[BPT], live[BPT];
            float wp[BPT];
#pragma unroll
            for (int b = 0; b < BPT; ++b) {
                const int li = jt * BPT + b;
                live[b] = li < nu;
                const int blk = blist[live[b] ? li : 0];
                sel[b] = live[b] && ((myw[blk >> 5] >> (blk & 31)) & 1u);
                wp[b] = (ORDER == 3 && live[b] && !sel[b]) ? __ldg(wrow + blk) : 0.f;
            }
            uint32_t sv[C::NK];
#pragma unroll
            for (int c = 0; c < C::NK / 32; ++c)
                tc::tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32 * c));
            tc::tmem_wait_ld();
            float cand[BPT], sbar[BPT], l2[BPT];
#pragma unroll
            for (int b = 0; b < BPT; ++b) {
                cand[b] = block_pass1<BS, ORDER>(sv + b * BS, sel[b], gate, ln_b, wp[b], sbar[b], l2[b]);
                if (!live[b]) cand[b] = -INFINITY;
            }
            float mc = cand[0];
#pragma unroll
            for (int b = 1; b < BPT; ++b) mc = fmaxf(mc, cand[b]);
            const bool raise = mc > m_run + 8.0f;
            const float scale = raise ? tc::ex2(m_run - mc) : 1.0f;
            if (raise) {
                dsum *= scale;
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
            float alpha[BPT], c0[BPT];
#pragma unroll
            for (int b = 0; b < BPT; ++b) {
                alpha[b] = 0.f;
                c0[b] = 0.f;
                if (live[b] && !sel[b]) {
                    alpha[b] = tc::ex2(l2[b] - m_run);
                    dsum = fmaf((float)BS, alpha[b], dsum);
                    c0[b] = alpha[b] * (1.0f - sbar[b]);
                }
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int col = half * 64 + c * 32;
                    const int b = col / BS;
                    uint32_t pk[16];
                    if (live[b]) {
                        dsum += chunk_pass2<ORDER>(sv + col, sel[b], m_run, alpha[b], c0[b], pk);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    }
                    tc::tmem_st16(s_addr + col / 2, pk);
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
                tc::mbar_arrive(bar((half == 0 ? B_PHALF : B_PFULL) + h));
            }
        }

        // ---- between the phases: O (phase-1 numerator) into registers as fp32 pairs
        uint64_t acc[D / 2];
#pragma unroll
        for (int e = 0; e < D / 2; ++e) acc[e] = 0ull;
        if (NT > 0 && tc::mbar_wait_warp(bar(B_OFULL + h), 0, aborted, status, kWaitLimitCycles)) {
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t raw[32];
                tc::tmem_ld32(o_addr + c * 32, raw);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    acc[c * 16 + e] = tc::f2_make(__uint_as_float(raw[2 * e]), __uint_as_float(raw[2 * e + 1]));
            }
        }
        tc::fence_before_sync();
        tc::mbar_arrive(bar(B_ODRAIN));

        // ---- phase 2: blocks unselected by every tile of the CTA
        for (int g = 0; !aborted && g < NI; ++g) {
            const int it = 2 * g + h, slot = it % C::NSLOT, use = it / C::NSLOT;
            const int vs = g % C::NV;
            if (!tc::mbar_wait_warp(bar(B_GFULL + slot), use & 1, aborted, status, kWaitLimitCycles)) break;
            if (!tc::mbar_wait_warp(bar(B_VSFULL + vs), (g / C::NV) & 1, aborted, status, kWaitLimitCycles)) break;
            // the phase is complete (lane 0 saw it); each thread's own test of it is its acquire
            (void)tc::mbar_try_wait(bar(B_VSFULL + vs), (g / C::NV) & 1);
            tc::fence_after_sync();
            const uint32_t gaddr = lane_base + (uint32_t)(slot * C::SLOT_STRIDE);
            uint32_t sc[16];  // the 16 centroid columns: high and low part of q . kbar_j, 8 apart
            tc::tmem_ld16(gaddr + C::AUG_ROW0, sc);
            tc::tmem_wait_ld();
            const float* vsm = reinterpret_cast<const float*>(smem + C::VS_OFF + vs * C::VS_BYTES);
#pragma unroll
            for (int b = 0; b < C::GB; ++b) {
                const int li = g * C::GB + b;
                const bool live = li < nn;
                const int blk = nlist[live ? li : 0];
                // q . kbar_j as q . (high part) + q . (low part), both from the MMA
                const float sb = __uint_as_float(sc[8 * b]) + __uint_as_float(sc[8 * b + 1]);
                const float wv = (ORDER == 3 && live) ? __ldg(wrow + blk) : 0.f;
                const float l2 = (sb + wv) * LOG2E;
                if (live && l2 > m_run + 8.0f) {
                    const float s2 = tc::ex2(m_run - l2);
                    const uint64_t s22 = tc::f2_make(s2, s2);
                    dsum *= s2;
#pragma unroll
                    for (int e = 0; e < D / 2; ++e) acc[e] = tc::f2_mul(acc[e], s22);
                    m_run = l2;
                }
                const float alpha = live ? tc::ex2(l2 - m_run) : 0.f;
                dsum = fmaf((float)BS, alpha, dsum);
                const uint64_t al2 = tc::f2_make(alpha, alpha);
                const float4* vrow = reinterpret_cast<const float4*>(vsm + b * D);
#pragma unroll
                for (int c = 0; c < D / 16; ++c) {
                    uint32_t gr[16];
                    tc::tmem_ld16(gaddr + (uint32_t)(b * D + c * 16), gr);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const float4 vv = vrow[c * 4 + e4];
                        const uint64_t g0 = tc::f2_add(
                            tc::f2_make(__uint_as_float(gr[4 * e4]), __uint_as_float(gr[4 * e4 + 1])),
                            tc::f2_make(vv.x, vv.y));
                        const uint64_t g1 = tc::f2_add(
                            tc::f2_make(__uint_as_float(gr[4 * e4 + 2]), __uint_as_float(gr[4 * e4 + 3])),
                            tc::f2_make(vv.z, vv.w));
                        acc[c * 8 + 2 * e4] = tc::f2_fma(al2, g0, acc[c * 8 + 2 * e4]);
                        acc[c * 8 + 2 * e4 + 1] = tc::f2_fma(al2, g1, acc[c * 8 + 2 * e4 + 1]);
                    }
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(bar(B_GEMPTY + slot));
            tc::mbar_arrive(bar(B_VSEMPTY + vs));
        }

        // ---- epilogue: o = N / D
        if (!aborted) {
            const float inv = 1.0f / dsum;
            // optional log-denominator ln D_t = m ln 2 + ln(dsum) (m in log2 units), for the backward
            if (lse && valid) lse[(size_t)bh * L + qrow] = fmaf(m_run, 0.6931471805599453f, logf(dsum));
            bf16* orow = out + ((size_t)bh * L + (valid ? qrow : 0)) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 x = tc::f2_split(acc[c * 16 + e]);
                    pk[e] = tc::pack_bf16x2(x.x * inv, x.y * inv);
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

// Host: tensor maps and launch of the statistics-form kernel.
//   hstat [BH, nblk, d, d] bf16 (row = value channel), kaug [BH, nblk, 8, d] bf16
//   (rows: bf16 high part of kbar_j, bf16 low part, six zero rows), vsum [BH, nblk, d]
//   fp32.  Requires L % 128 == 0 and BH * nblk * d < 2^31 (checked by the caller).
// order 3 = first order + the pooled w matrix `wmat`.
inline pisa_status run_attn_stc(const void* q, const void* k, const void* v, const void* hstat, const void* kaug,
                                const float* vsum, const uint32_t* mask, void* out, long BH, int L, int d, int B,
                                int nblk, int words, int order, int gate, const float* wmat, unsigned* status,
                                cudaStream_t s, std::string* err, float* lse = nullptr) {
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
    CUtensorMap mq, mk, mv, mh, ma;
    if (!make(&mq, q, BH * L, 128) || !make(&mk, k, BH * L, B) || !make(&mv, v, BH * L, B) ||
        !make(&mh, hstat, BH * nblk * d, d) || !make(&ma, kaug, BH * nblk * 8, 8)) {
        *err = "cuTensorMapEncodeTiled failed for the statistics-form kernel";
        return PISA_ERR_CUDA;
    }
    dim3 grid((unsigned)((L + 255) / 256), (unsigned)BH);
    cudaError_t e = cudaSuccess;
    int regs = 0;
#define PISA_STC_LAUNCH(DD, BB, OO)                                                                              \
    if (d == DD && B == BB && order == OO) {                                                                     \
        auto kern = attn_stc_kernel<DD, BB, OO>;                                                                 \
        cudaFuncAttributes fa;                                                                                   \
        e = cudaFuncGetAttributes(&fa, kern);                                                                    \
        regs = fa.numRegs;                                                                                       \
        if (e == cudaSuccess && regs >= (int)kStcRegsLaunch)                                                     \
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StcCfg<DD, BB>::SMEM); \
        if (e == cudaSuccess && regs >= (int)kStcRegsLaunch) {                                                   \
            kern<<<grid, kStcThreads, StcCfg<DD, BB>::SMEM, s>>>(mq, mk, mv, mh, ma, mask, vsum, (bf16*)out, L,    \
                                                                 nblk, words, gate, logf((float)B), wmat, status, \
                                                                 lse);                                            \
            e = cudaGetLastError();                                                                              \
        }                                                                                                        \
    } else
    PISA_STC_LAUNCH(64, 64, 1)
    PISA_STC_LAUNCH(64, 64, 3)
    PISA_STC_LAUNCH(64, 128, 1)
    PISA_STC_LAUNCH(64, 128, 3)
    PISA_STC_LAUNCH(128, 64, 1)
    PISA_STC_LAUNCH(128, 64, 3)
    PISA_STC_LAUNCH(128, 128, 1)
    PISA_STC_LAUNCH(128, 128, 3) {
        *err = "no statistics-form tensor-core kernel for this d/B/order";
        return PISA_ERR_UNSUPPORTED;
    }
#undef PISA_STC_LAUNCH
    if (e == cudaSuccess && regs < (int)kStcRegsLaunch) {
        // setmaxnreg.inc would wait for registers the CTA was never given
        *err = "attn_stc_kernel was built with " + std::to_string(regs) + " registers a thread, the register split "
               "needs " + std::to_string(kStcRegsLaunch);
        return PISA_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) {
        *err = std::string("attn_stc_kernel launch: ") + cudaGetErrorString(e);
        return PISA_ERR_CUDA;
    }
    return PISA_OK;
}

}  // namespace pisa
