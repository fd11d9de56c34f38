// Block statistics on tcgen05 tensor cores (bf16 inputs).
//
// Per key block j (PISA paper, section 3.4 and Figure 3, the prepare phase;
// "Sparse Linear Attention" blog, sections "Sparse Linear Attention" and "Going
// Further: Adding the Second-Order Term (PWT)"):
//   kbar_j = (1/B) sum_n k_n          canonical fp32 pairwise tree (CUDA cores)
//   vsum_j = sum_n v_n                fp32 (CUDA cores)
//   H_j    = sum_n v_n (k_n - kbar_j)^T = V_j^T K_j - vsum_j kbar_j^T
//   C_j    = (1/B) sum_n (k_n - kbar_j)(k_n - kbar_j)^T = (1/B) K_j^T K_j - kbar_j kbar_j^T
// The two Gram products run on the tensor cores straight from the token tiles:
// V_j^T and K_j^T are read as MN-major A operands, K_j as the MN-major B
// operand (both K-dimensions are the B tokens), fp32 accumulation in TMEM; the
// rank-1 corrections and the 1/B are applied in fp32 in the epilogue.  For
// d = 64 the A operand is [V_j^T ; K_j^T] stacked to M = 128, so one MMA gives
// H_j (rows 0-63) and the uncentred C_j (rows 64-127).
//
// With kaug non-null it also writes, per block, the eight bf16 rows the
// statistics-form tensor-core kernel appends to H_j as extra B-operand rows:
// row 0 = bf16(kbar_j) (round to nearest), row 1 = bf16(kbar_j - row 0), rows
// 2-7 = 0, so that one MMA gives q . kbar_j as two columns to within about
// 2^-16 of the fp32 centroid.
//
// Persistent CTAs (one per SM), each looping over blocks: see stats_tc_kernel.
#pragma once

#include <cudaTypedefs.h>

#include <string>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace pisa {

template <int D, int BS, int ORDER>
struct StatsTcCfg {
    static constexpr uint32_t BOX_BYTES = BS * 128;             // BS rows x 64 bf16 columns
    static constexpr uint32_t TILE_BYTES = (D / 64) * BOX_BYTES;
    static constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;     // V tile, then K tile ([V ; K] for d = 64)
    // output staging: per epilogue warp one 32-row x 64-column box (4 KB) per matrix and column half
    static constexpr int HALVES = D / 64;                       // 64-column boxes per output row
    static constexpr int OUT_BOXES = ((D == 128 && ORDER == 2) ? 2 : 1) * HALVES;
    static constexpr uint32_t OUT_BYTES = 4 * OUT_BOXES * 4096;
    static constexpr int NSTG_FIT = (int)((204800 - OUT_BYTES) / STAGE_BYTES);
    static constexpr int NSTG = NSTG_FIT < 6 ? NSTG_FIT : 6;
    static constexpr uint32_t OUT_OFF = NSTG * STAGE_BYTES;
    static constexpr uint32_t BAR_OFF = OUT_OFF + OUT_BYTES;
    // FULL, EMPTY per stage; MMADONE, EPIDONE per TMEM buffer; KBREADY, KBFREE per
    // kbar/vsum buffer; DONE
    static constexpr uint32_t NBAR = 2 * NSTG + 8 + 1;
    static constexpr uint32_t KB_OFF = BAR_OFF + NBAR * 8 + 8;  // fp32 kbar[2][D], vsum[2][D]
    static constexpr uint32_t SMEM = KB_OFF + 4 * D * 4 + 1024;
    static constexpr int THREADS = 320;  // producer, MMA, four column-sum warps, four epilogue warps
    static_assert(NSTG >= 2, "the statistics kernel needs two stages");
    static_assert(KB_OFF % 16 == 0, "kbar and vsum are read as 16-byte vectors");
    static_assert(SMEM <= 232448, "shared memory over the per-CTA limit");
};

template <int D, int ORDER>
constexpr uint32_t stats_tmem_cols() { return D == 128 ? (ORDER == 2 ? 256u : 128u) : 64u; }

// bf16 element (n, c) of a tile staged by TMA with 128-byte swizzle in boxes of
// 64 columns: 16-byte chunk index XOR (row mod 8).
template <int BS>
__device__ __forceinline__ float swz_elem(const uint8_t* tile, int n, int c) {
    const int box = c >> 6, cc = c & 63;
    const int chunk = (cc >> 3) ^ (n & 7);
    const bf16* p = reinterpret_cast<const bf16*>(tile + box * (BS * 128) + n * 128 + chunk * 16) + (cc & 7);
    return __bfloat162float(*p);
}

template <int BITS>
__host__ __device__ constexpr int bit_reverse(int x) {
    int r = 0;
    for (int b = 0; b < BITS; ++b) r |= ((x >> b) & 1) << (BITS - 1 - b);
    return r;
}

// Column c of a swizzled B-row tile (see swz_elem), summed two ways: `tree` the canonical
// pairwise tree (rows n and n + B/2 first, then n and n + B/4, ...), evaluated depth-first
// over the rows in bit-reversed order, where each level combines adjacent partial sums, so
// at most log2(B) + 1 of them are live; `serial` in row order.  The tree is the same
// sequence of separately rounded adds as tree_sum<B>.
template <int BS, bool TREE>
__device__ __forceinline__ float column_sum(const uint8_t* tile, int c) {
    constexpr int LB = (BS == 128) ? 7 : 6;
    const uint8_t* col = tile + (c >> 6) * (BS * 128) + (c & 7) * 2;
    const int c8 = (c & 63) >> 3;
    if constexpr (TREE) {
        float st[LB + 1];
#pragma unroll
        for (int p = 0; p < BS; ++p) {
            const int n = bit_reverse<LB>(p);
            float v = __bfloat162float(*reinterpret_cast<const bf16*>(col + n * 128 + ((c8 ^ (n & 7)) << 4)));
            int lvl = 0;
#pragma unroll
            for (int t = 0; t < LB; ++t) {
                if (((p >> t) & 1) && lvl == t) {
                    v = __fadd_rn(st[t], v);
                    lvl = t + 1;
                }
            }
            st[lvl] = v;
        }
        return st[LB];
    } else {
        float sv = 0.f;
#pragma unroll
        for (int n = 0; n < BS; ++n)
            sv += __bfloat162float(*reinterpret_cast<const bf16*>(col + n * 128 + ((c8 ^ (n & 7)) << 4)));
        return sv;
    }
}

// Persistent: CTA c takes the blocks c, c + grid, c + 2 grid, ... of the flattened
// (bh, j) index.  Warp 0 streams K_j and V_j through NSTG TMA stages; warp 1 runs the
// Gram MMAs into two TMEM buffers (block i into buffer i % 2); warps 2-5 take the
// column sums of block i from its stage (k-bar by the canonical tree, the value sums in
// row order) into a double-buffered kbar/vsum pair; warps 6-9 run the epilogue of block
// i from TMEM: warp w reads lane quarter w % 4, applies the rank-1 corrections, rounds
// to bf16 into its own 128-byte-swizzled staging boxes (32 rows x 64 columns each; the
// row-per-thread 16-byte stores hit distinct banks) and writes each box with one TMA
// store.  The two roles overlap: the column sums of block i + 1 run beside the epilogue
// of block i.  A stage is free again once its MMA has completed and the column-sum warps
// have read it; a TMEM buffer once the epilogue has read it; a kbar/vsum buffer once the
// epilogue of its block is done; a staging box once the warp's previous store has read it.
template <int D, int BS, int ORDER>
__global__ void __launch_bounds__(320, 1) stats_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                          const __grid_constant__ CUtensorMap tm_v,
                                                          const __grid_constant__ CUtensorMap tm_h,
                                                          const __grid_constant__ CUtensorMap tm_c,
                                                          float* __restrict__ kbar, float* __restrict__ vsum,
                                                          bf16* __restrict__ kaug, int nblk, int L, long total,
                                                          unsigned* status) {
    using C = StatsTcCfg<D, BS, ORDER>;
    // M = 128 always (d = 64 stacks V and K); N = d; both operands MN-major
    constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                               ((uint32_t)(D >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    constexpr uint32_t TCOLS = stats_tmem_cols<D, ORDER>();  // one buffer
    constexpr long long LIMIT = 2000000000ll;
    constexpr int NSUM = 4, NEPI = 4;  // column-sum warps, epilogue warps
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_addr(smem);
    auto bar = [&](int i) { return sbase + C::BAR_OFF + 8u * (uint32_t)i; };
    const int B_FULL = 0, B_EMPTY = C::NSTG, B_MMADONE = 2 * C::NSTG, B_EPIDONE = B_MMADONE + 2,
              B_KBREADY = B_EPIDONE + 2, B_KBFREE = B_KBREADY + 2, B_DONE = B_KBFREE + 2;
    uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + C::NBAR * 8);
    float* kbs = (float*)(smem + C::KB_OFF);  // [2][D]
    float* vss = kbs + 2 * D;                 // [2][D]
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    bool aborted = false;
    // number of blocks this CTA processes
    const long first = blockIdx.x, stride = gridDim.x;
    const int nmine = first < total ? (int)((total - 1 - first) / stride + 1) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSTG; ++s) {
            tc::mbar_init(bar(B_FULL + s), 1);
            tc::mbar_init(bar(B_EMPTY + s), 1 + NSUM);  // the MMA's commit + the column-sum warps
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(bar(B_MMADONE + b), 1);
            tc::mbar_init(bar(B_EPIDONE + b), NEPI);
            tc::mbar_init(bar(B_KBREADY + b), NSUM);  // the block's kbar/vsum are in kbs/vss
            tc::mbar_init(bar(B_KBFREE + b), NEPI);   // the epilogue has read them
        }
        tc::mbar_init(bar(B_DONE), 1);
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), 2 * TCOLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tc::tma_prefetch(&tm_k);
            tc::tma_prefetch(&tm_v);
            int last = -1;
            for (int i = 0; i < nmine; ++i) {
                const int s = i % C::NSTG, u = i / C::NSTG;
                if (u > 0 && !tc::mbar_wait(bar(B_EMPTY + s), (u - 1) & 1, aborted, status, LIMIT)) break;
                const long blk = first + (long)i * stride;
                const int bh = (int)(blk / nblk), j = (int)(blk % nblk);
                const int row = bh * L + j * BS;
                const uint32_t st = sbase + s * C::STAGE_BYTES;
                tc::mbar_expect_tx(bar(B_FULL + s), C::STAGE_BYTES);
                for (int b = 0; b < D / 64; ++b) {
                    tc::tma_load_2d(st + b * C::BOX_BYTES, &tm_v, bar(B_FULL + s), b * 64, row);
                    tc::tma_load_2d(st + C::TILE_BYTES + b * C::BOX_BYTES, &tm_k, bar(B_FULL + s), b * 64, row);
                }
                last = i;
            }
            if (aborted) {
                // let the copies already issued land before the CTA exits
                for (int i = (last - C::NSTG + 1 > 0 ? last - C::NSTG + 1 : 0); i <= last; ++i) {
                    bool a2 = false;
                    tc::mbar_wait(bar(B_FULL + i % C::NSTG), (i / C::NSTG) & 1, a2, status, LIMIT);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            for (int i = 0; i < nmine; ++i) {
                const int s = i % C::NSTG, u = i / C::NSTG, buf = i & 1, ub = i >> 1;
                if (!tc::mbar_wait(bar(B_FULL + s), u & 1, aborted, status, LIMIT)) break;
                if (ub > 0 && !tc::mbar_wait(bar(B_EPIDONE + buf), (ub - 1) & 1, aborted, status, LIMIT)) break;
                tc::fence_after_sync();
                const uint32_t sa = sbase + s * C::STAGE_BYTES;
                const uint32_t dt = tmem + (uint32_t)(buf * TCOLS);
#pragma unroll
                for (int kk = 0; kk < BS / 16; ++kk) {
                    const uint32_t off = kk * 16 * 128;  // 16 tokens further along K
                    // H_raw (d = 128), or [H_raw ; C_raw] (d = 64): A = V^T (stacked with K^T)
                    const uint64_t a_v = tc::sdesc_sw128(sa + off, C::BOX_BYTES, 1024);
                    const uint64_t b_k = tc::sdesc_sw128(sa + C::TILE_BYTES + off, C::BOX_BYTES, 1024);
                    tc::mma_ss(dt, a_v, b_k, IDESC, kk > 0);
                    if (D == 128 && ORDER == 2) tc::mma_ss(dt + 128, b_k, b_k, IDESC, kk > 0);
                }
                tc::mma_commit(bar(B_MMADONE + buf));
                tc::mma_commit(bar(B_EMPTY + s));
            }
            // every MMA issued by this thread has completed before TMEM is freed
            tc::mma_commit(bar(B_DONE));
            bool a2 = false;
            tc::mbar_wait(bar(B_DONE), 0, a2, status, LIMIT);
        }
    } else if (warp < 2 + NSUM) {
        // ---------------------------------------------------------------- column sums
        // d = 128: thread ct takes k column ct and v column ct; d = 64: threads 0-63 the k
        // columns, 64-127 the v columns
        const int ct = threadIdx.x - 64;  // 0 .. 127
        for (int i = 0; i < nmine; ++i) {
            const int s = i % C::NSTG, u = i / C::NSTG, kb = i & 1, ukb = i >> 1;
            const long blk = first + (long)i * stride;
            if (!tc::mbar_wait_warp(bar(B_FULL + s), u & 1, aborted, status, LIMIT)) break;
            // the phase is complete (lane 0 saw it); each thread's own test of it is its acquire
            // of the stage's bytes
            (void)tc::mbar_try_wait(bar(B_FULL + s), u & 1);
            // the kbar/vsum buffer is free once the epilogue of block i - 2 has read it
            if (ukb > 0 && !tc::mbar_wait_warp(bar(B_KBFREE + kb), (ukb - 1) & 1, aborted, status, LIMIT)) break;
            const uint8_t* st = smem + s * C::STAGE_BYTES;
            const size_t so = (size_t)blk * D;
            const bool do_k = (D == 128) || ct < D;
            const bool do_v = (D == 128) || ct >= D;
            const int c = (D == 128) ? ct : (ct & (D - 1));
            if (do_k) {
                const float m = __fmul_rn(column_sum<BS, true>(st + C::TILE_BYTES, c), 1.0f / (float)BS);
                kbs[kb * D + c] = m;
                kbar[so + c] = m;
                if (kaug) {
                    bf16* ka = kaug + (size_t)blk * 8 * D + c;
                    const bf16 hi = __float2bfloat16_rn(m);
                    ka[0] = hi;
                    ka[D] = __float2bfloat16_rn(m - __bfloat162float(hi));
#pragma unroll
                    for (int rr = 2; rr < 8; ++rr) ka[rr * D] = __float2bfloat16_rn(0.f);
                }
            }
            if (do_v) {
                const float sv = column_sum<BS, false>(st, c);
                vss[kb * D + c] = sv;
                vsum[so + c] = sv;
            }
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(bar(B_EMPTY + s));     // this warp no longer reads the stage
                tc::mbar_arrive(bar(B_KBREADY + kb));  // and its kbar/vsum columns are in kbs/vss
            }
        }
    } else {
        // ----------------------------------------------------------------- epilogue
        const int quarter = warp % 4;  // TMEM lane quarter of this warp
        const int r = quarter * 32 + lane;  // TMEM lane = output row
        const float inv_b = 1.0f / (float)BS;
        // for d = 64, rows 0-63 are H_j and rows 64-127 the uncentred C_j
        const bool is_h = (D == 128) || (quarter < 2);
        const bool writes = is_h || ORDER == 2;
        const int ar = (D == 128) ? r : (r & 63);  // row of the output matrix
        const uint32_t stg = sbase + C::OUT_OFF + (uint32_t)(warp - 2 - NSUM) * (C::OUT_BOXES * 4096u);
        for (int i = 0; i < nmine; ++i) {
            const int buf = i & 1, ub = i >> 1, kb = i & 1;
            const long blk = first + (long)i * stride;
            if (!tc::mbar_wait_warp(bar(B_KBREADY + kb), ub & 1, aborted, status, LIMIT)) break;
            // kbs/vss were written by the column-sum threads: each thread's own test is its acquire
            (void)tc::mbar_try_wait(bar(B_KBREADY + kb), ub & 1);
            if (!tc::mbar_wait_warp(bar(B_MMADONE + buf), ub & 1, aborted, status, LIMIT)) break;
            tc::fence_after_sync();
            if (writes) {
                // the staging boxes are free once this warp's previous stores have read them
                if (lane == 0) tc::bulk_wait_read<0>();
                __syncwarp();
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * TCOLS);
                const float* kbp = kbs + kb * D;
                const float* vsp = vss + kb * D;
#pragma unroll
                for (int part = 0; part < C::OUT_BOXES / C::HALVES; ++part) {
                    const bool h_here = (D == 128) ? (part == 0) : is_h;
                    const float rv = h_here ? vsp[ar] : kbp[ar];
#pragma unroll
                    for (int hf = 0; hf < C::HALVES; ++hf) {
                        const uint32_t box = stg + (uint32_t)(part * C::HALVES + hf) * 4096u;
#pragma unroll
                        for (int c0 = 0; c0 < 64; c0 += 32) {
                            uint32_t raw[32];
                            tc::tmem_ld32(taddr + (uint32_t)(part * 128 + hf * 64 + c0), raw);
                            tc::tmem_wait_ld();
                            uint32_t pk[16];
                            const float4* kb4 = reinterpret_cast<const float4*>(kbp + hf * 64 + c0);
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) {
                                const float4 kv = kb4[e4];  // kbar of the four columns (a broadcast read)
                                const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                                for (int e2 = 0; e2 < 2; ++e2) {
                                    const int e = 2 * e4 + e2;
                                    float x0 = __uint_as_float(raw[2 * e]), x1 = __uint_as_float(raw[2 * e + 1]);
                                    if (h_here) {
                                        x0 = fmaf(-rv, kk[2 * e2], x0);
                                        x1 = fmaf(-rv, kk[2 * e2 + 1], x1);
                                    } else {
                                        x0 = fmaf(-rv, kk[2 * e2], x0 * inv_b);
                                        x1 = fmaf(-rv, kk[2 * e2 + 1], x1 * inv_b);
                                    }
                                    pk[e] = tc::pack_bf16x2(x0, x1);
                                }
                            }
                            // row `lane` of the box, 16-byte chunks c0/8 .. c0/8 + 3, swizzled
                            const uint32_t rowa = box + (uint32_t)lane * 128u;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const uint32_t chunk = (uint32_t)((c0 / 8 + e) ^ (lane & 7));
                                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowa + chunk * 16u),
                                             "r"(pk[4 * e]), "r"(pk[4 * e + 1]), "r"(pk[4 * e + 2]), "r"(pk[4 * e + 3])
                                             : "memory");
                            }
                        }
                    }
                }
            }
            // TMEM and kbs/vss are read: the MMA may reuse the buffer, the column sums the pair
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(bar(B_EPIDONE + buf));
                tc::mbar_arrive(bar(B_KBFREE + kb));
            }
            if (writes) {
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int y = (int)((long)blk * D + (ar - lane));  // first row of the boxes
#pragma unroll
                    for (int part = 0; part < C::OUT_BOXES / C::HALVES; ++part) {
                        const bool h_here = (D == 128) ? (part == 0) : is_h;
#pragma unroll
                        for (int hf = 0; hf < C::HALVES; ++hf)
                            tc::tma_store_2d(h_here ? &tm_h : &tm_c, stg + (uint32_t)(part * C::HALVES + hf) * 4096u,
                                             hf * 64, y);
                    }
                    tc::bulk_commit();
                }
            }
        }
        // the stores have landed before the CTA exits
        if (lane == 0) tc::bulk_wait<0>();
        __syncwarp();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 2 * TCOLS);
    }
}

inline pisa_status run_stats_tc(const void* k, const void* v, float* kbar, float* vsum, void* hstat, void* cov,
                                void* kaug, long BH, int L, int d, int B, int nblk, int order, unsigned* status,
                                cudaStream_t s, std::string* err) {
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
    if (order == 2 && !cov) {
        *err = "the second-order statistics need a C_j buffer";
        return PISA_ERR_INVALID_ARG;
    }
    // K and V as loaded (box 64 columns x B rows); H_j and C_j as stored (box 64 columns x
    // 32 rows of the [BH nblk d, d] matrices)
    CUtensorMap maps[4];
    const long mrows = BH * (long)nblk * d;
    struct MapSpec {
        const void* p;
        long rows;
        uint32_t box_rows;
    } specs[4] = {{k, BH * (long)L, (uint32_t)B}, {v, BH * (long)L, (uint32_t)B}, {hstat, mrows, 32u},
                  {cov ? cov : hstat, mrows, 32u}};
    for (int t = 0; t < 4; ++t) {
        cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)specs[t].rows};
        cuuint64_t gstride[1] = {(cuuint64_t)d * 2};
        cuuint32_t box[2] = {64, specs[t].box_rows};
        cuuint32_t estride[2] = {1, 1};
        CUresult cr = encode(&maps[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(specs[t].p), gdim,
                             gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS) {
            *err = "cuTensorMapEncodeTiled failed (" + std::to_string((int)cr) + ")";
            return PISA_ERR_CUDA;
        }
    }
    // persistent: one CTA per SM (fewer when there are fewer blocks)
    static int nsm = 0;
    if (!nsm) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0) nsm = 148;
    }
    const long total = BH * (long)nblk;
    dim3 grid((unsigned)(total < nsm ? total : nsm));
    cudaError_t e = cudaSuccess;
#define PISA_STATS_TC(DD, BB, OO)                                                                             \
    if (d == DD && B == BB && order == OO) {                                                                  \
        using SC = StatsTcCfg<DD, BB, OO>;                                                                    \
        auto kern = stats_tc_kernel<DD, BB, OO>;                                                              \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SC::SMEM);           \
        if (e == cudaSuccess) {                                                                               \
            kern<<<grid, SC::THREADS, SC::SMEM, s>>>(maps[0], maps[1], maps[2], maps[3], kbar, vsum,           \
                                                     (bf16*)kaug, nblk, L, total, status);                    \
            e = cudaGetLastError();                                                                           \
        }                                                                                                     \
    } else
    PISA_STATS_TC(64, 64, 1)
    PISA_STATS_TC(64, 64, 2)
    PISA_STATS_TC(64, 128, 1)
    PISA_STATS_TC(64, 128, 2)
    PISA_STATS_TC(128, 64, 1)
    PISA_STATS_TC(128, 64, 2)
    PISA_STATS_TC(128, 128, 1)
    PISA_STATS_TC(128, 128, 2) {
        *err = "no tensor-core statistics kernel for this d/B/order";
        return PISA_ERR_UNSUPPORTED;
    }
#undef PISA_STATS_TC
    if (e != cudaSuccess) {
        *err = std::string("stats_tc_kernel launch: ") + cudaGetErrorString(e);
        return PISA_ERR_CUDA;
    }
    return PISA_OK;
}

}  // namespace pisa
