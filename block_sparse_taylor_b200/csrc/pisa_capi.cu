// C ABI of the piecewise sparse attention library (declared in include/pisa.h).
//
// Host side only: argument validation, workspace layout, kernel selection and
// launches.  Every launch is asynchronous on the caller's stream; nothing here
// allocates device memory or synchronises, except pisa_poll_device_status.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <string>

#include "../../include/pisa.h"
#include "common.cuh"
#include "stats.cuh"
#include "select.cuh"
#include "attn_stats.cuh"
#include "attn_tc.cuh"
#include "stats_tc.cuh"
#include "hybrid_prep.cuh"
#include "attn_hybrid.cuh"
#include "attn_stc.cuh"
#include "route.cuh"
#include "backward.cuh"
#include "backward_tc.cuh"
#include "selftest.cuh"

using pisa::bf16;

namespace {

thread_local std::string g_last_error;

// One status word per device (module-scope device variable).
__device__ unsigned int g_device_status;

pisa_status fail(pisa_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
pisa_status fail(pisa_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

pisa_status cuda_fail(cudaError_t e, const char* where) {
    return fail(PISA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

unsigned int* device_status_ptr() {
    static unsigned int* cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        cache[dev] = (unsigned int*)p;
    }
    return cache[dev];
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
size_t esize(pisa_dtype t) { return t == PISA_BF16 ? 2 : 4; }

struct Dims {
    long BH, L, d, B, nblk, words;
};

// Shape validation common to every entry point.
pisa_status check_dims(int batch, int heads, int L, int d, int B, int order, pisa_dtype dtype, Dims* out) {
    if (batch <= 0 || heads <= 0 || L <= 0 || d <= 0 || B <= 0)
        return fail(PISA_ERR_INVALID_ARG, "batch, heads, L, d and B must be positive");
    if (dtype != PISA_F32 && dtype != PISA_BF16) return fail(PISA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (order < 0 || order > 2) return fail(PISA_ERR_INVALID_ARG, "order must be 0, 1 or 2 (got %d)", order);
    if (L % B) return fail(PISA_ERR_INVALID_ARG, "L (%d) must be a multiple of B (%d)", L, B);
    if (d != 64 && d != 128) return fail(PISA_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
    if (B != 64 && B != 128) return fail(PISA_ERR_UNSUPPORTED, "B must be 64 or 128 (got %d)", B);
    const long nblk = L / B;
    if (nblk > 4096) return fail(PISA_ERR_UNSUPPORTED, "L/B must be <= 4096 (got %ld)", nblk);
    out->BH = (long)batch * heads;
    out->L = L;
    out->d = d;
    out->B = B;
    out->nblk = nblk;
    out->words = (nblk + 31) / 32;
    return PISA_OK;
}

// Device arrays that kernels move with 16-byte vector accesses or TMA must be
// 16-byte aligned.  Contiguous tensors from an allocator always are; a view at an
// odd element offset may not be, and would fault the kernel instead of failing here.
pisa_status check_align16(const char* where, std::initializer_list<const void*> ptrs) {
    for (const void* p : ptrs)
        if (p && (uintptr_t)p % 16)
            return fail(PISA_ERR_INVALID_ARG, "%s: device arrays must be 16-byte aligned", where);
    return PISA_OK;
}

struct StatsLayout {
    size_t kbar, vsum, hstat, cov, kaug, total;
};

// kaug (the bf16 high/low split of the centroids) exists for bf16, order >= 1
bool has_kaug(int order, pisa_dtype dtype) { return dtype == PISA_BF16 && order >= 1; }

StatsLayout stats_layout(const Dims& g, int order, pisa_dtype dtype) {
    StatsLayout s{};
    size_t o = 0;
    s.kbar = o;
    o += align_up(sizeof(float) * g.BH * g.nblk * g.d);
    s.vsum = o;
    o += align_up(sizeof(float) * g.BH * g.nblk * g.d);
    s.hstat = o;
    if (order >= 1) o += align_up(esize(dtype) * g.BH * g.nblk * g.d * g.d);
    s.cov = o;
    if (order == 2) o += align_up(esize(dtype) * g.BH * g.nblk * g.d * g.d);
    s.kaug = o;
    if (has_kaug(order, dtype)) o += align_up(2 * g.BH * g.nblk * 8 * g.d);
    s.total = o;
    return s;
}

// ---------------------------------------------------------------------------
// launch helpers (template dispatch over dtype, d, B)
// ---------------------------------------------------------------------------

template <typename F>
pisa_status dispatch(pisa_dtype dtype, int d, int B, F&& f) {
#define PISA_CASE(T, DD, BB) \
    if (d == DD && B == BB) return f(T(), std::integral_constant<int, DD>(), std::integral_constant<int, BB>());
    if (dtype == PISA_BF16) {
        PISA_CASE(bf16, 64, 64)
        PISA_CASE(bf16, 64, 128)
        PISA_CASE(bf16, 128, 64)
        PISA_CASE(bf16, 128, 128)
    } else {
        PISA_CASE(float, 64, 64)
        PISA_CASE(float, 64, 128)
        PISA_CASE(float, 128, 64)
        PISA_CASE(float, 128, 128)
    }
#undef PISA_CASE
    return fail(PISA_ERR_UNSUPPORTED, "no kernel for d=%d B=%d", d, B);
}

template <typename K>
pisa_status set_smem(K kernel, size_t bytes) {
    static int max_optin = -1;
    if (max_optin < 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            max_optin = 0;
    }
    if ((long)bytes > max_optin)
        return fail(PISA_ERR_UNSUPPORTED, "kernel needs %zu bytes of shared memory (device allows %d)", bytes,
                    max_optin);
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    return PISA_OK;
}

pisa_status launch_check(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, what);
    return PISA_OK;
}

pisa_status run_centroids(const void* k, float* kbar, const Dims& g, pisa_dtype dtype, cudaStream_t s) {
    return dispatch(dtype, (int)g.d, (int)g.B, [&](auto t, auto dd, auto bb) {
        using T = decltype(t);
        constexpr int D = decltype(dd)::value, BS = decltype(bb)::value;
        const size_t smem = sizeof(T) * BS * D;
        auto kern = pisa::centroid_kernel<T, D, BS>;
        pisa_status r = set_smem(kern, smem);
        if (r != PISA_OK) return r;
        dim3 grid((unsigned)g.nblk, (unsigned)g.BH);
        kern<<<grid, 128, smem, s>>>((const T*)k, kbar, (int)g.L, (int)g.nblk);
        return launch_check("centroid_kernel");
    });
}

pisa_status run_stats(const void* k, const void* v, const pisa_stats_t* st, const Dims& g, cudaStream_t s) {
    if (st->dtype == PISA_BF16 && st->order >= 1) {
        // bf16: the Gram products H_j and C_j on the tensor cores
        unsigned int* status = device_status_ptr();
        if (!status) return fail(PISA_ERR_CUDA, "cannot resolve the device status word");
        return pisa::run_stats_tc(k, v, st->kbar, st->vsum, st->hstat, st->cov, st->kaug, g.BH, (int)g.L, (int)g.d,
                                  (int)g.B, (int)g.nblk, st->order, status, s, &g_last_error);
    }
    return dispatch(st->dtype, (int)g.d, (int)g.B, [&](auto t, auto dd, auto bb) {
        using T = decltype(t);
        constexpr int D = decltype(dd)::value, BS = decltype(bb)::value;
        const size_t smem = sizeof(float) * ((size_t)2 * BS * (D + 1) + D);
        auto kern = pisa::stats_simt_kernel<T, D, BS>;
        pisa_status r = set_smem(kern, smem);
        if (r != PISA_OK) return r;
        dim3 grid((unsigned)g.nblk, (unsigned)g.BH);
        kern<<<grid, 256, smem, s>>>((const T*)k, (const T*)v, st->kbar, st->vsum, (T*)st->hstat, (T*)st->cov,
                                     (int)g.L, (int)g.nblk, st->order);
        return launch_check("stats_simt_kernel");
    });
}

pisa_status run_select(const void* q, const float* kbar, const Dims& g, pisa_dtype dtype, int K, int32_t* idx,
                       uint32_t* mask, cudaStream_t s, const float* bias = nullptr, float* scores = nullptr) {
    return dispatch(dtype, (int)g.d, (int)g.B, [&](auto t, auto dd, auto bb) {
        using T = decltype(t);
        constexpr int D = decltype(dd)::value, BS = decltype(bb)::value;
        const int QT = pisa::select_tiles_per_cta<D>((int)g.nblk);
        const size_t smem = pisa::select_smem_bytes<D>(QT, (int)g.nblk);
        auto kern = pisa::select_kernel<T, D, BS>;
        pisa_status r = set_smem(kern, smem);
        if (r != PISA_OK) return r;
        dim3 grid((unsigned)((g.nblk + QT - 1) / QT), (unsigned)g.BH);
        kern<<<grid, pisa::SelectCfg<D>::THREADS, smem, s>>>((const T*)q, kbar, (int)g.L, (int)g.nblk, K,
                                                              (int)g.words, QT, idx, mask, bias, scores);
        return launch_check("select_kernel");
    });
}

// Covariance-aware routing bias ln(||H_j||_F + eps), [BH, nblk] fp32.
pisa_status run_route_bias(const void* k, const void* v, const float* kbar, const Dims& g, pisa_dtype dtype,
                           float eps, float* bias, cudaStream_t s) {
    return dispatch(dtype, (int)g.d, (int)g.B, [&](auto t, auto dd, auto bb) {
        using T = decltype(t);
        constexpr int D = decltype(dd)::value, BS = decltype(bb)::value;
        const size_t smem = pisa::RouteCfg<D, BS>::SMEM;
        auto kern = pisa::route_bias_kernel<T, D, BS>;
        pisa_status r = set_smem(kern, smem);
        if (r != PISA_OK) return r;
        dim3 grid((unsigned)g.nblk, (unsigned)g.BH);
        kern<<<grid, pisa::RouteCfg<D, BS>::THREADS, smem, s>>>((const T*)k, (const T*)v, kbar, (int)g.L,
                                                                 (int)g.nblk, eps, bias);
        return launch_check("route_bias_kernel");
    });
}

pisa_status run_attn_stats(const void* q, const void* k, const void* v, const pisa_stats_t* st,
                           const uint32_t* mask, void* out, const Dims& g, int order, int gate,
                           cudaStream_t s, const float* wmat = nullptr, float* lse = nullptr) {
    return dispatch(st->dtype, (int)g.d, (int)g.B, [&](auto t, auto dd, auto bb) {
        using T = decltype(t);
        constexpr int D = decltype(dd)::value, BS = decltype(bb)::value;
        const size_t smem = pisa::AttnStatsSmem<T, D, BS>::bytes;
        auto kern = pisa::attn_stats_kernel<T, D, BS>;
        pisa_status r = set_smem(kern, smem);
        if (r != PISA_OK) return r;
        constexpr int parts = BS / pisa::AttnStatsSmem<T, D, BS>::RQ;  // CTAs per query tile
        dim3 grid((unsigned)(g.nblk * parts), (unsigned)g.BH);
        kern<<<grid, 256, smem, s>>>((const T*)q, (const T*)k, (const T*)v, st->kbar, st->vsum,
                                     (const T*)st->hstat, (const T*)st->cov, mask, (T*)out, (int)g.L,
                                     (int)g.nblk, (int)g.words, order, gate, logf((float)g.B), wmat, lse);
        return launch_check("attn_stats_kernel");
    });
}

// PWT's cheap second-order term: per-block channel variances of k, tile means
// of q^2, then the gated [query tile x block] matrix w.
pisa_status run_wpool(const void* q, const void* k, const Dims& g, pisa_dtype dtype, int gate, float* var, float* q2,
                      float* wmat, cudaStream_t s) {
    return dispatch(dtype, (int)g.d, (int)g.B, [&](auto t, auto dd, auto bb) {
        using T = decltype(t);
        constexpr int D = decltype(dd)::value, BS = decltype(bb)::value;
        const size_t smem = sizeof(T) * BS * D;
        auto kv = pisa::colstat_kernel<T, D, BS, 1>;
        auto kq = pisa::colstat_kernel<T, D, BS, 2>;
        pisa_status r = set_smem(kv, smem);
        if (r != PISA_OK) return r;
        r = set_smem(kq, smem);
        if (r != PISA_OK) return r;
        dim3 grid((unsigned)g.nblk, (unsigned)g.BH);
        kv<<<grid, 128, smem, s>>>((const T*)k, var, (int)g.L, (int)g.nblk);
        kq<<<grid, 128, smem, s>>>((const T*)q, q2, (int)g.L, (int)g.nblk);
        pisa::wpool_kernel<D><<<grid, 256, 0, s>>>(q2, var, wmat, (int)g.nblk, gate, logf((float)g.B));
        return launch_check("pooled-w kernels");
    });
}

// ---------------------------------------------------------------------------
// workspace layout of pisa_attention
// ---------------------------------------------------------------------------
struct WsLayout {
    size_t stats, mask, idx, bias, total;
    StatsLayout sl;
    size_t kbar_bf, vsum_bf, hbar_acc, hbar_bf;  // hybrid path only
    size_t var, q2, wmat;                        // order 2: PWT's pooled w (used with the pooled flag)
};

WsLayout ws_layout(const Dims& g, int K, int order, pisa_dtype dtype, pisa_path path) {
    WsLayout w{};
    if (path == PISA_PATH_RECOMPUTE_TC || path == PISA_PATH_HYBRID_TC) {
        // The token-form and hybrid paths need only the fp32 centroids (for the selection).
        w.sl = StatsLayout{};
        w.sl.total = align_up(sizeof(float) * g.BH * g.nblk * g.d);
    } else if (path == PISA_PATH_STATS_TC) {
        // kbar, vsum, H_j and the centroid split; the pooled second order needs no C_j
        w.sl = stats_layout(g, 1, dtype);
    } else {
        w.sl = stats_layout(g, order, dtype);
    }
    size_t o = 0;
    w.stats = o;
    o += w.sl.total;
    w.mask = o;
    o += align_up(sizeof(uint32_t) * g.BH * g.nblk * g.words);
    w.idx = o;
    o += align_up(sizeof(int32_t) * g.BH * g.nblk * (K > 0 ? K : 1));
    w.bias = o;  // routing bias (used with PISA_FLAG_COV_ROUTE)
    o += align_up(sizeof(float) * g.BH * g.nblk);
    if (path == PISA_PATH_HYBRID_TC) {
        w.kbar_bf = o;
        o += align_up(2 * g.BH * g.nblk * g.d);
        w.vsum_bf = o;
        o += align_up(2 * g.BH * g.nblk * g.d);
        w.hbar_acc = o;  // H-bar's per-chunk slots, reduced in a fixed order
        o += align_up(4 * g.BH * (size_t)pisa::hybrid_prep_nchunk(g.BH, (int)g.nblk) * g.d * g.d);
        w.hbar_bf = o;
        o += align_up(2 * g.BH * g.d * g.d);
    }
    if (order == 2) {
        w.var = o;
        o += align_up(4 * g.BH * g.nblk * g.d);
        w.q2 = o;
        o += align_up(4 * g.BH * g.nblk * g.d);
        w.wmat = o;
        o += align_up(4 * g.BH * g.nblk * g.nblk);
    }
    w.total = o;
    return w;
}

// The hybrid supports orders 0 and 1, and order 2 in PWT's pooled form only.
bool hybrid_path_available(const Dims& g, pisa_dtype dtype, int order) {
    return dtype == PISA_BF16 && pisa::attn_tc_supported((int)g.d, (int)g.B) && g.L % 128 == 0 && order <= 2 &&
           g.BH * g.L <= 0x7fffffffL;
}

bool tc_path_available(const Dims& g, pisa_dtype dtype) {
    return dtype == PISA_BF16 && pisa::attn_tc_supported((int)g.d, (int)g.B) && g.L % 128 == 0 &&
           g.BH * g.L <= 0x7fffffffL;
}

// The statistics form on the tensor cores: first order (or the pooled second order).
bool stc_path_available(const Dims& g, pisa_dtype dtype, int order, bool pooled) {
    return tc_path_available(g, dtype) && g.BH * g.nblk * g.d <= 0x7fffffffL &&
           (order == 1 || (order == 2 && pooled));
}

// Executed FLOPs per query row of the statistics-form tensor-core kernel with the union of
// the CTA's selections at its bound min(nblk, (256/B) K), and of the token form (4 L d).
double stc_flops_per_row(const Dims& g, int K) {
    const long nqt = 256 / g.B, bpt = 128 / g.B, gb = g.d == 64 ? 2 : 1;
    const long u = std::min<long>(g.nblk, nqt * (long)K);
    const long nut = (u + bpt - 1) / bpt, ni = (g.nblk - u + gb - 1) / gb;
    return 4.0 * g.d * 128.0 * nut + 2.0 * g.d * (gb * g.d + 16) * ni;
}
double token_flops_per_row(const Dims& g) { return 4.0 * g.d * g.L; }

// On the tensor cores, the association that executes fewer FLOPs (the statistics
// form only for order 1: at order 2 its C_j contraction doubles it); else the
// statistics path on CUDA cores.
pisa_path resolve(const Dims& g, int K, int order, pisa_dtype dtype) {
    if (!tc_path_available(g, dtype)) return PISA_PATH_STATS;
    if (stc_path_available(g, dtype, order, false) && stc_flops_per_row(g, K) < token_flops_per_row(g))
        return PISA_PATH_STATS_TC;
    return PISA_PATH_RECOMPUTE_TC;
}

// ---------------------------------------------------------------------------
// backward pass: workspace layout and launches
// ---------------------------------------------------------------------------
struct BwdLayout {
    size_t kbar, bias, mask, mstat, dinv, delta, lse;
    // order 2 only: PWT's pooled w and its gradient (var, q2 [BH, nblk, d]; wmat, wsum
    // [BH, nblk, nblk]; wpart [BH, L / 32, nblk])
    size_t var, q2, wmat, wsum, wpart, total;
};

BwdLayout bwd_layout(const Dims& g, int order) {
    BwdLayout w{};
    size_t o = 0;
    w.kbar = o;
    o += align_up(sizeof(float) * g.BH * g.nblk * g.d);
    w.bias = o;
    o += align_up(sizeof(float) * g.BH * g.nblk);
    w.mask = o;
    o += align_up(sizeof(uint32_t) * g.BH * g.nblk * g.words);
    w.mstat = o;
    o += align_up(sizeof(float) * g.BH * g.L);
    w.dinv = o;
    o += align_up(sizeof(float) * g.BH * g.L);
    w.delta = o;
    o += align_up(sizeof(float) * g.BH * g.L);
    w.lse = o;
    o += align_up(sizeof(float) * g.BH * g.L);
    w.var = w.q2 = w.wmat = w.wsum = w.wpart = 0;
    if (order == 2) {
        w.var = o;
        o += align_up(sizeof(float) * g.BH * g.nblk * g.d);
        w.q2 = o;
        o += align_up(sizeof(float) * g.BH * g.nblk * g.d);
        w.wmat = o;
        o += align_up(sizeof(float) * g.BH * g.nblk * g.nblk);
        w.wsum = o;
        o += align_up(sizeof(float) * g.BH * g.nblk * g.nblk);
        w.wpart = o;
        o += align_up(sizeof(float) * g.BH * (g.L / 32) * g.nblk);
    }
    w.total = o;
    return w;
}

// The backward on tcgen05 (bf16, the tensor-core shapes): delta (and, without the forward's
// lse, the row statistics turned into lse), then the dq and dk/dv kernels.
pisa_status run_backward_tc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                            const uint32_t* mask, const Dims& g, int order, int gate, const float* lse_in,
                            float* mst, float* dinv, float* del, float* lse_ws, float* dq, float* dk, float* dv,
                            cudaStream_t s, const float* wmat = nullptr, float* wpart = nullptr) {
    // order 3: the first order with PWT's pooled w (wmat), its gradient gathered in wpart
    unsigned int* status = device_status_ptr();
    if (!status) return fail(PISA_ERR_CUDA, "cannot resolve the device status word");
    const long rows = g.BH * g.L;
    const float* lse = lse_in;
    if (!lse_in) {
        // m_t, 1/D_t and delta_t from the row-statistics kernel, then lse = m - ln(1/D)
        pisa_status r = dispatch(PISA_BF16, (int)g.d, (int)g.B, [&](auto t, auto dd, auto bb) {
            using T = decltype(t);
            constexpr int D = decltype(dd)::value, BS = decltype(bb)::value;
            using C = pisa::bwd::Cfg<T, D, BS>;
            auto k1 = pisa::bwd::bwd_rowstat_kernel<T, D, BS>;
            pisa_status rr = set_smem(k1, C::ROWSTAT_SMEM);
            if (rr != PISA_OK) return rr;
            const dim3 gq((unsigned)(g.L / pisa::bwd::kQT), (unsigned)g.BH);
            k1<<<gq, 128, C::ROWSTAT_SMEM, s>>>((const T*)q, (const T*)k, (const T*)o, (const T*)dO, mask, (int)g.L,
                                                (int)g.nblk, (int)g.words, order, gate, mst, dinv, del);
            return launch_check("bwd_rowstat_kernel");
        });
        if (r != PISA_OK) return r;
        pisa::bwdtc::bwd_lse_kernel<<<(unsigned)((rows + 255) / 256 < 4096 ? (rows + 255) / 256 : 4096), 256, 0, s>>>(
            mst, dinv, rows, lse_ws);
        r = launch_check("bwd_lse_kernel");
        if (r != PISA_OK) return r;
        lse = lse_ws;
    } else {
        const unsigned nb = (unsigned)((rows + 7) / 8);
        if (g.d == 64)
            pisa::bwdtc::bwd_delta_kernel<64><<<nb, 256, 0, s>>>((const bf16*)o, (const bf16*)dO, rows, del);
        else
            pisa::bwdtc::bwd_delta_kernel<128><<<nb, 256, 0, s>>>((const bf16*)o, (const bf16*)dO, rows, del);
        pisa_status r = launch_check("bwd_delta_kernel");
        if (r != PISA_OK) return r;
    }
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess || !fn)
            return fail(PISA_ERR_CUDA, "cuTensorMapEncodeTiled not available");
        encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    }
    CUtensorMap maps[4];
    const void* ptrs[4] = {q, k, v, dO};
    for (int t = 0; t < 4; ++t) {
        cuuint64_t gdim[2] = {(cuuint64_t)g.d, (cuuint64_t)rows};
        cuuint64_t gstride[1] = {(cuuint64_t)g.d * 2};
        cuuint32_t box[2] = {64, 128};
        cuuint32_t estride[2] = {1, 1};
        if (encode(&maps[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptrs[t]), gdim, gstride, box,
                   estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return fail(PISA_ERR_CUDA, "cuTensorMapEncodeTiled failed for the backward kernels");
    }
    const dim3 grid((unsigned)(g.L / 128), (unsigned)g.BH);
    cudaError_t e = cudaSuccess;
    bool found = false;
#define PISA_BWD_TC(DD, BB, OO)                                                                                   \
    if (!found && g.d == DD && g.B == BB && order == OO) {                                                        \
        found = true;                                                                                             \
        auto kq = pisa::bwdtc::bwd_dq_tc_kernel<DD, BB, OO>;                                                      \
        auto kk = pisa::bwdtc::bwd_dkdv_tc_kernel<DD, BB, OO>;                                                    \
        e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pisa::bwdtc::DqCfg<DD>::SMEM); \
        if (e == cudaSuccess)                                                                                     \
            e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize,                             \
                                     (int)pisa::bwdtc::DkvCfg<DD, BB>::SMEM);                                         \
        if (e == cudaSuccess) {                                                                                   \
            kq<<<grid, pisa::bwdtc::kThreads, pisa::bwdtc::DqCfg<DD>::SMEM, s>>>(                                 \
                maps[0], maps[1], maps[2], maps[3], mask, lse, del, dq, (int)g.L, (int)g.nblk, (int)g.words, gate,  \
                status, wmat, wpart);                                                                             \
            e = cudaGetLastError();                                                                               \
        }                                                                                                         \
        if (e == cudaSuccess) {                                                                                   \
            kk<<<grid, pisa::bwdtc::kThreads, pisa::bwdtc::DkvCfg<DD, BB>::SMEM, s>>>(                                \
                maps[0], maps[1], maps[2], maps[3], mask, lse, del, dk, dv, (int)g.L, (int)g.nblk, (int)g.words,    \
                gate, status, wmat);                                                                              \
            e = cudaGetLastError();                                                                               \
        }                                                                                                         \
    }
    PISA_BWD_TC(64, 64, 0)
    PISA_BWD_TC(64, 64, 1)
    PISA_BWD_TC(64, 64, 2)
    PISA_BWD_TC(64, 128, 0)
    PISA_BWD_TC(64, 128, 1)
    PISA_BWD_TC(64, 128, 2)
    PISA_BWD_TC(128, 64, 0)
    PISA_BWD_TC(128, 64, 1)
    PISA_BWD_TC(128, 64, 2)
    PISA_BWD_TC(128, 128, 0)
    PISA_BWD_TC(128, 128, 1)
    PISA_BWD_TC(128, 128, 2)
    PISA_BWD_TC(64, 64, 3)
    PISA_BWD_TC(64, 128, 3)
    PISA_BWD_TC(128, 64, 3)
    PISA_BWD_TC(128, 128, 3)
#undef PISA_BWD_TC
    if (!found) return fail(PISA_ERR_UNSUPPORTED, "no tensor-core backward kernel for this d/B/order");
    if (e != cudaSuccess) return cuda_fail(e, "backward tensor-core kernels");
    return PISA_OK;
}

pisa_status run_backward(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const uint32_t* mask, const Dims& g, pisa_dtype dtype, int order, int gate, float* mst,
                         float* dinv, float* del, float* dq, float* dk, float* dv, cudaStream_t s) {
    return dispatch(dtype, (int)g.d, (int)g.B, [&](auto t, auto dd, auto bb) {
        using T = decltype(t);
        constexpr int D = decltype(dd)::value, BS = decltype(bb)::value;
        using C = pisa::bwd::Cfg<T, D, BS>;
        auto k1 = pisa::bwd::bwd_rowstat_kernel<T, D, BS>;
        auto k2 = pisa::bwd::bwd_dq_kernel<T, D, BS>;
        auto k3 = pisa::bwd::bwd_dkdv_kernel<T, D, BS>;
        pisa_status r = set_smem(k1, C::ROWSTAT_SMEM);
        if (r == PISA_OK) r = set_smem(k2, C::DQ_SMEM);
        if (r == PISA_OK) r = set_smem(k3, C::DKDV_SMEM);
        if (r != PISA_OK) return r;
        const int L = (int)g.L, nblk = (int)g.nblk, words = (int)g.words;
        const dim3 gq((unsigned)(g.L / pisa::bwd::kQT), (unsigned)g.BH);
        k1<<<gq, 128, C::ROWSTAT_SMEM, s>>>((const T*)q, (const T*)k, (const T*)o, (const T*)dO, mask, L, nblk, words,
                                            order, gate, mst, dinv, del);
        r = launch_check("bwd_rowstat_kernel");
        if (r != PISA_OK) return r;
        k2<<<gq, 128, C::DQ_SMEM, s>>>((const T*)q, (const T*)k, (const T*)v, (const T*)dO, mask, L, nblk, words,
                                       order, gate, mst, dinv, del, dq);
        r = launch_check("bwd_dq_kernel");
        if (r != PISA_OK) return r;
        const dim3 gk((unsigned)g.nblk, (unsigned)g.BH);
        k3<<<gk, 2 * BS, C::DKDV_SMEM, s>>>((const T*)q, (const T*)k, (const T*)v, (const T*)dO, mask, L, nblk,
                                            words, order, gate, mst, dinv, del, dk, dv);
        return launch_check("bwd_dkdv_kernel");
    });
}

pisa_status check_stats(const pisa_stats_t* st, Dims* g) {
    if (!st) return fail(PISA_ERR_INVALID_ARG, "null pisa_stats_t");
    pisa_status r = check_dims(st->batch, st->heads, st->L, st->d, st->B, st->order, st->dtype, g);
    if (r != PISA_OK) return r;
    if (st->nblk != g->nblk) return fail(PISA_ERR_INVALID_ARG, "pisa_stats_t.nblk inconsistent with L/B");
    if (!st->kbar || !st->vsum) return fail(PISA_ERR_INVALID_ARG, "pisa_stats_t: null kbar or vsum");
    if (st->order >= 1 && !st->hstat) return fail(PISA_ERR_INVALID_ARG, "pisa_stats_t: null hstat for order >= 1");
    if (st->order == 2 && !st->cov) return fail(PISA_ERR_INVALID_ARG, "pisa_stats_t: null cov for order 2");
    if (st->kaug && !has_kaug(st->order, st->dtype))
        return fail(PISA_ERR_INVALID_ARG, "pisa_stats_t: kaug is for bf16 statistics of order >= 1 only");
    return PISA_OK;
}

}  // namespace

extern "C" {

const char* pisa_version(void) { return "pisa-b200 0.2"; }

const char* pisa_last_error(void) { return g_last_error.c_str(); }

size_t pisa_stats_bytes(int batch, int heads, int L, int d, int B, int order, pisa_dtype dtype) {
    Dims g;
    if (check_dims(batch, heads, L, d, B, order, dtype, &g) != PISA_OK) return 0;
    return stats_layout(g, order, dtype).total;
}

pisa_status pisa_stats_bind(pisa_stats_t* st, void* buf, size_t bytes, int batch, int heads, int L, int d, int B,
                            int order, pisa_dtype dtype) {
    if (!st || !buf) return fail(PISA_ERR_INVALID_ARG, "pisa_stats_bind: null st or buf");
    if ((uintptr_t)buf % kAlign) return fail(PISA_ERR_INVALID_ARG, "pisa_stats_bind: buf must be 256-byte aligned");
    Dims g;
    pisa_status r = check_dims(batch, heads, L, d, B, order, dtype, &g);
    if (r != PISA_OK) return r;
    StatsLayout s = stats_layout(g, order, dtype);
    if (bytes < s.total)
        return fail(PISA_ERR_INVALID_ARG, "pisa_stats_bind: buffer of %zu bytes, need %zu", bytes, s.total);
    char* b = (char*)buf;
    st->batch = batch;
    st->heads = heads;
    st->L = L;
    st->d = d;
    st->B = B;
    st->nblk = (int)g.nblk;
    st->order = order;
    st->dtype = dtype;
    st->kbar = (float*)(b + s.kbar);
    st->vsum = (float*)(b + s.vsum);
    st->hstat = order >= 1 ? (void*)(b + s.hstat) : nullptr;
    st->cov = order == 2 ? (void*)(b + s.cov) : nullptr;
    st->kaug = has_kaug(order, dtype) ? (void*)(b + s.kaug) : nullptr;
    return PISA_OK;
}

pisa_status pisa_stats(const void* k, const void* v, const pisa_stats_t* st, void* stream) {
    Dims g;
    pisa_status r = check_stats(st, &g);
    if (r != PISA_OK) return r;
    if (!k || !v) return fail(PISA_ERR_INVALID_ARG, "pisa_stats: null k or v");
    r = check_align16("pisa_stats", {k, v, st->kbar, st->vsum, st->hstat, st->cov, st->kaug});
    if (r != PISA_OK) return r;
    return run_stats(k, v, st, g, (cudaStream_t)stream);
}

pisa_status pisa_select(const void* q, const pisa_stats_t* st, int K, int32_t* idx, uint32_t* mask, void* stream) {
    Dims g;
    if (!st) return fail(PISA_ERR_INVALID_ARG, "null pisa_stats_t");
    pisa_status r = check_dims(st->batch, st->heads, st->L, st->d, st->B, 0, st->dtype, &g);
    if (r != PISA_OK) return r;
    if (!st->kbar) return fail(PISA_ERR_INVALID_ARG, "pisa_select: null kbar");
    if (!q) return fail(PISA_ERR_INVALID_ARG, "pisa_select: null q");
    if (K < 0 || K > g.nblk) return fail(PISA_ERR_INVALID_ARG, "K must be in [0, %ld] (got %d)", g.nblk, K);
    if (!idx && !mask) return fail(PISA_ERR_INVALID_ARG, "pisa_select: idx and mask both null");
    r = check_align16("pisa_select", {q, st->kbar});
    if (r != PISA_OK) return r;
    return run_select(q, st->kbar, g, st->dtype, K, K > 0 ? idx : nullptr, mask, (cudaStream_t)stream);
}

pisa_status pisa_select_biased(const void* q, const pisa_stats_t* st, int K, const float* bias, int32_t* idx,
                               uint32_t* mask, void* stream) {
    Dims g;
    if (!st) return fail(PISA_ERR_INVALID_ARG, "null pisa_stats_t");
    pisa_status r = check_dims(st->batch, st->heads, st->L, st->d, st->B, 0, st->dtype, &g);
    if (r != PISA_OK) return r;
    if (!st->kbar) return fail(PISA_ERR_INVALID_ARG, "pisa_select_biased: null kbar");
    if (!q) return fail(PISA_ERR_INVALID_ARG, "pisa_select_biased: null q");
    if (K < 0 || K > g.nblk) return fail(PISA_ERR_INVALID_ARG, "K must be in [0, %ld] (got %d)", g.nblk, K);
    if (!idx && !mask) return fail(PISA_ERR_INVALID_ARG, "pisa_select_biased: idx and mask both null");
    r = check_align16("pisa_select_biased", {q, st->kbar});
    if (r != PISA_OK) return r;
    return run_select(q, st->kbar, g, st->dtype, K, K > 0 ? idx : nullptr, mask, (cudaStream_t)stream, bias);
}

pisa_status pisa_select_scores(const void* q, const pisa_stats_t* st, const float* bias, float* scores,
                               void* stream) {
    Dims g;
    if (!st) return fail(PISA_ERR_INVALID_ARG, "null pisa_stats_t");
    pisa_status r = check_dims(st->batch, st->heads, st->L, st->d, st->B, 0, st->dtype, &g);
    if (r != PISA_OK) return r;
    if (!st->kbar || !q || !scores) return fail(PISA_ERR_INVALID_ARG, "pisa_select_scores: null pointer");
    r = check_align16("pisa_select_scores", {q, st->kbar});
    if (r != PISA_OK) return r;
    return run_select(q, st->kbar, g, st->dtype, 0, nullptr, nullptr, (cudaStream_t)stream, bias, scores);
}

pisa_status pisa_route_bias(const void* k, const void* v, const float* kbar, int batch, int heads, int L, int d,
                            pisa_dtype dtype, int B, float eps, float* bias, void* stream) {
    Dims g;
    pisa_status r = check_dims(batch, heads, L, d, B, 0, dtype, &g);
    if (r != PISA_OK) return r;
    if (!k || !v || !kbar || !bias) return fail(PISA_ERR_INVALID_ARG, "pisa_route_bias: null pointer");
    r = check_align16("pisa_route_bias", {k, v, kbar});
    if (r != PISA_OK) return r;
    if (!(eps >= 1e-30f && eps <= 1e30f))
        return fail(PISA_ERR_INVALID_ARG, "pisa_route_bias: eps must be in [1e-30, 1e30] (got %g)", (double)eps);
    return run_route_bias(k, v, kbar, g, dtype, eps, bias, (cudaStream_t)stream);
}

int pisa_resolve_path(int batch, int heads, int L, int d, int B, int K, int order, pisa_dtype dtype) {
    Dims g;
    if (check_dims(batch, heads, L, d, B, order, dtype, &g) != PISA_OK) return -1;
    if (K < 0 || K > g.nblk) return -1;
    return (int)resolve(g, K, order, dtype);
}

size_t pisa_workspace_bytes_ex(int batch, int heads, int L, int d, int B, int K, int order, pisa_dtype dtype,
                               pisa_path path) {
    Dims g;
    if (check_dims(batch, heads, L, d, B, order, dtype, &g) != PISA_OK) return 0;
    if (K < 0 || K > g.nblk) return 0;
    if (path == PISA_PATH_AUTO) path = resolve(g, K, order, dtype);
    if (path == PISA_PATH_RECOMPUTE_TC && !tc_path_available(g, dtype)) return 0;
    if (path == PISA_PATH_HYBRID_TC && !hybrid_path_available(g, dtype, order)) return 0;
    // order 2 runs on this path only with the pooled w, so size it for that
    if (path == PISA_PATH_STATS_TC && !stc_path_available(g, dtype, order, order == 2)) return 0;
    if (path != PISA_PATH_STATS && path != PISA_PATH_RECOMPUTE_TC && path != PISA_PATH_HYBRID_TC &&
        path != PISA_PATH_STATS_TC)
        return 0;
    return ws_layout(g, K, order, dtype, path).total;
}

size_t pisa_workspace_bytes(int batch, int heads, int L, int d, int B, int K, int order, pisa_dtype dtype) {
    return pisa_workspace_bytes_ex(batch, heads, L, d, B, K, order, dtype, PISA_PATH_AUTO);
}

}  // extern "C"

namespace {

// pisa_attention_ex with an optional per-row log-denominator output (lse may be null).
pisa_status attention_impl(const void* q, const void* k, const void* v, int batch, int heads, int L, int d,
                           pisa_dtype dtype, int B, int K, int order, int gate_w, pisa_path path, void* out,
                           float* lse, void* workspace, size_t ws_bytes, void* stream) {
    Dims g;
    pisa_status r = check_dims(batch, heads, L, d, B, order, dtype, &g);
    if (r != PISA_OK) return r;
    if (K < 0 || K > g.nblk) return fail(PISA_ERR_INVALID_ARG, "K must be in [0, %ld] (got %d)", g.nblk, K);
    if (!q || !k || !v || !out) return fail(PISA_ERR_INVALID_ARG, "pisa_attention: null q, k, v or out");
    r = check_align16("pisa_attention", {q, k, v, out});
    if (r != PISA_OK) return r;
    if (!workspace) return fail(PISA_ERR_INVALID_ARG, "pisa_attention: null workspace");
    if ((uintptr_t)workspace % kAlign)
        return fail(PISA_ERR_INVALID_ARG, "pisa_attention: workspace must be 256-byte aligned");
    if (path == PISA_PATH_AUTO) path = resolve(g, K, order, dtype);
    if (path == PISA_PATH_RECOMPUTE_TC && !tc_path_available(g, dtype))
        return fail(PISA_ERR_UNSUPPORTED, "tensor-core path needs bf16, d and B in {64, 128}, L %% 128 == 0");
    if (path == PISA_PATH_HYBRID_TC && !hybrid_path_available(g, dtype, order))
        return fail(PISA_ERR_UNSUPPORTED, "hybrid path needs bf16, d and B in {64, 128}, L %% 128 == 0");
    const int gate = gate_w & PISA_FLAG_GATE_W;
    const bool pooled = (gate_w & PISA_FLAG_POOLED_W) != 0;
    const bool route = (gate_w & PISA_FLAG_COV_ROUTE) != 0;
    if (path == PISA_PATH_HYBRID_TC && order == 2 && !pooled)
        return fail(PISA_ERR_UNSUPPORTED, "the hybrid's second order needs the pooled w (PISA_FLAG_POOLED_W)");
    if (path == PISA_PATH_HYBRID_TC && lse)
        return fail(PISA_ERR_UNSUPPORTED, "no log-denominator output on the hybrid path");
    if (lse && (uintptr_t)lse % 4) return fail(PISA_ERR_INVALID_ARG, "lse must be 4-byte aligned");
    if (path == PISA_PATH_STATS_TC && !stc_path_available(g, dtype, order, pooled))
        return fail(PISA_ERR_UNSUPPORTED,
                    "statistics-form tensor-core path needs bf16, d and B in {64, 128}, L %% 128 == 0 and order 1 "
                    "(order 2 only with PISA_FLAG_POOLED_W)");
    if (path != PISA_PATH_STATS && path != PISA_PATH_RECOMPUTE_TC && path != PISA_PATH_HYBRID_TC &&
        path != PISA_PATH_STATS_TC)
        return fail(PISA_ERR_INVALID_ARG, "unknown path %d", (int)path);
    const WsLayout w = ws_layout(g, K, order, dtype, path);
    if (ws_bytes < w.total)
        return fail(PISA_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", ws_bytes, w.total);
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    pisa_stats_t st{};
    st.batch = batch;
    st.heads = heads;
    st.L = L;
    st.d = d;
    st.B = B;
    st.nblk = (int)g.nblk;
    st.dtype = dtype;
    st.order = (path == PISA_PATH_RECOMPUTE_TC || path == PISA_PATH_HYBRID_TC) ? 0
               : (path == PISA_PATH_STATS_TC)                                ? 1
                                                                             : order;
    st.kbar = (float*)(ws + w.stats + w.sl.kbar);
    st.vsum = (path == PISA_PATH_STATS || path == PISA_PATH_STATS_TC) ? (float*)(ws + w.stats + w.sl.vsum) : nullptr;
    st.hstat = st.order >= 1 ? (void*)(ws + w.stats + w.sl.hstat) : nullptr;
    st.cov = st.order == 2 ? (void*)(ws + w.stats + w.sl.cov) : nullptr;
    st.kaug = (path == PISA_PATH_STATS_TC) ? (void*)(ws + w.stats + w.sl.kaug) : nullptr;
    uint32_t* mask = (uint32_t*)(ws + w.mask);
    int32_t* idx = (int32_t*)(ws + w.idx);
    float* rbias = route ? (float*)(ws + w.bias) : nullptr;

    float* wmat = nullptr;
    if (order == 2 && pooled) {
        wmat = (float*)(ws + w.wmat);
        r = run_wpool(q, k, g, dtype, gate, (float*)(ws + w.var), (float*)(ws + w.q2), wmat, s);
        if (r != PISA_OK) return r;
    }
    const int korder = (order == 2 && pooled) ? 3 : order;  // kernel order code (3 = pooled w)
    if (path == PISA_PATH_HYBRID_TC) {
        unsigned int* status = device_status_ptr();
        if (!status) return fail(PISA_ERR_CUDA, "cannot resolve the device status word");
        bf16* kbar_bf = (bf16*)(ws + w.kbar_bf);
        bf16* vsum_bf = (bf16*)(ws + w.vsum_bf);
        float* hacc = (float*)(ws + w.hbar_acc);
        bf16* hbf = (bf16*)(ws + w.hbar_bf);
        r = pisa::run_hybrid_prep(k, v, st.kbar, kbar_bf, vsum_bf, hacc, hbf, g.BH, (int)g.L, (int)g.d, (int)g.B,
                                  (int)g.nblk, status, s, &g_last_error);
        if (r != PISA_OK) return r;
        if (route) {
            r = run_route_bias(k, v, st.kbar, g, dtype, PISA_ROUTE_EPS, rbias, s);
            if (r != PISA_OK) return r;
        }
        r = run_select(q, st.kbar, g, dtype, K, K > 0 ? idx : nullptr, mask, s, rbias);
        if (r != PISA_OK) return r;
        return pisa::run_attn_hybrid(q, k, v, kbar_bf, vsum_bf, hbf, mask, out, g.BH, (int)g.L, (int)g.d, (int)g.B,
                                     (int)g.nblk, (int)g.words, korder, wmat, status, s, &g_last_error);
    }
    if (path == PISA_PATH_RECOMPUTE_TC) {
        r = run_centroids(k, st.kbar, g, dtype, s);
        if (r != PISA_OK) return r;
    } else {
        r = run_stats(k, v, &st, g, s);
        if (r != PISA_OK) return r;
    }
    if (route) {
        r = run_route_bias(k, v, st.kbar, g, dtype, PISA_ROUTE_EPS, rbias, s);
        if (r != PISA_OK) return r;
    }
    r = run_select(q, st.kbar, g, dtype, K, K > 0 ? idx : nullptr, mask, s, rbias);
    if (r != PISA_OK) return r;
    if (path == PISA_PATH_RECOMPUTE_TC) {
        unsigned int* status = device_status_ptr();
        if (!status) return fail(PISA_ERR_CUDA, "cannot resolve the device status word");
        return pisa::run_attn_tc(q, k, v, mask, out, g.BH, (int)g.L, (int)g.d, (int)g.B, (int)g.nblk,
                                 (int)g.words, korder, gate, wmat, status, s, &g_last_error, lse);
    }
    if (path == PISA_PATH_STATS_TC) {
        unsigned int* status = device_status_ptr();
        if (!status) return fail(PISA_ERR_CUDA, "cannot resolve the device status word");
        return pisa::run_attn_stc(q, k, v, st.hstat, st.kaug, st.vsum, mask, out, g.BH, (int)g.L, (int)g.d, (int)g.B,
                                  (int)g.nblk, (int)g.words, korder, gate, wmat, status, s, &g_last_error, lse);
    }
    return run_attn_stats(q, k, v, &st, mask, out, g, order, gate, s, wmat, lse);
}

}  // namespace

extern "C" {

pisa_status pisa_attention_ex(const void* q, const void* k, const void* v, int batch, int heads, int L, int d,
                              pisa_dtype dtype, int B, int K, int order, int gate_w, pisa_path path, void* out,
                              void* workspace, size_t ws_bytes, void* stream) {
    return attention_impl(q, k, v, batch, heads, L, d, dtype, B, K, order, gate_w, path, out, nullptr, workspace,
                          ws_bytes, stream);
}

pisa_status pisa_attention_lse(const void* q, const void* k, const void* v, int batch, int heads, int L, int d,
                               pisa_dtype dtype, int B, int K, int order, int gate_w, pisa_path path, void* out,
                               float* lse, void* workspace, size_t ws_bytes, void* stream) {
    if (!lse) return fail(PISA_ERR_INVALID_ARG, "pisa_attention_lse: null lse");
    return attention_impl(q, k, v, batch, heads, L, d, dtype, B, K, order, gate_w, path, out, lse, workspace,
                          ws_bytes, stream);
}

pisa_status pisa_attention(const void* q, const void* k, const void* v, int batch, int heads, int L, int d,
                           pisa_dtype dtype, int B, int K, int order, void* out, void* workspace, size_t ws_bytes,
                           void* stream) {
    return pisa_attention_ex(q, k, v, batch, heads, L, d, dtype, B, K, order, 1, PISA_PATH_AUTO, out, workspace,
                             ws_bytes, stream);
}

size_t pisa_backward_workspace_bytes(int batch, int heads, int L, int d, int B, int K, int order, pisa_dtype dtype) {
    Dims g;
    if (check_dims(batch, heads, L, d, B, order, dtype, &g) != PISA_OK) return 0;
    if (K < 0 || K > g.nblk || g.BH > 65535) return 0;
    return bwd_layout(g, order).total;
}

}  // extern "C"

namespace {

pisa_status backward_impl(const void* q, const void* k, const void* v, const void* o, const void* dO, int batch,
                          int heads, int L, int d, pisa_dtype dtype, int B, int K, int order, int flags,
                          const float* lse, float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes,
                          void* stream) {
    Dims g;
    pisa_status r = check_dims(batch, heads, L, d, B, order, dtype, &g);
    if (r != PISA_OK) return r;
    if (K < 0 || K > g.nblk) return fail(PISA_ERR_INVALID_ARG, "K must be in [0, %ld] (got %d)", g.nblk, K);
    if (g.BH > 65535) return fail(PISA_ERR_UNSUPPORTED, "batch * heads must be <= 65535 (got %ld)", g.BH);
    if (flags & ~(PISA_FLAG_GATE_W | PISA_FLAG_POOLED_W | PISA_FLAG_COV_ROUTE))
        return fail(PISA_ERR_INVALID_ARG, "pisa_attention_backward: unknown flag bits 0x%x", flags);
    const bool pooled = (flags & PISA_FLAG_POOLED_W) != 0;
    if (pooled && order != 2)
        return fail(PISA_ERR_INVALID_ARG, "pisa_attention_backward: the pooled w is an order-2 option");
    if (pooled && !tc_path_available(g, dtype))
        return fail(PISA_ERR_UNSUPPORTED,
                    "pisa_attention_backward: the pooled-w backward runs on the tensor-core path (bf16, d and B in "
                    "{64, 128}, L a multiple of 128)");
    if (pooled && !lse)
        return fail(PISA_ERR_UNSUPPORTED,
                    "pisa_attention_backward: the pooled-w backward takes the forward's lse "
                    "(pisa_attention_backward_lse)");
    if (!q || !k || !v || !o || !dO || !dq || !dk || !dv)
        return fail(PISA_ERR_INVALID_ARG, "pisa_attention_backward: null pointer");
    const void* in16[5] = {q, k, v, o, dO};
    for (const void* p : in16)
        if ((uintptr_t)p % 16) return fail(PISA_ERR_INVALID_ARG, "pisa_attention_backward: inputs must be 16-byte aligned");
    if ((uintptr_t)dq % 8 || (uintptr_t)dk % 8 || (uintptr_t)dv % 8)
        return fail(PISA_ERR_INVALID_ARG, "pisa_attention_backward: dq, dk, dv must be 8-byte aligned");
    if (!workspace) return fail(PISA_ERR_INVALID_ARG, "pisa_attention_backward: null workspace");
    if ((uintptr_t)workspace % kAlign)
        return fail(PISA_ERR_INVALID_ARG, "pisa_attention_backward: workspace must be 256-byte aligned");
    const BwdLayout w = bwd_layout(g, order);
    if (ws_bytes < w.total)
        return fail(PISA_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", ws_bytes, w.total);
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    float* kbar = (float*)(ws + w.kbar);
    uint32_t* mask = (uint32_t*)(ws + w.mask);
    float* rbias = (flags & PISA_FLAG_COV_ROUTE) ? (float*)(ws + w.bias) : nullptr;
    r = run_centroids(k, kbar, g, dtype, s);
    if (r != PISA_OK) return r;
    if (rbias) {
        r = run_route_bias(k, v, kbar, g, dtype, PISA_ROUTE_EPS, rbias, s);
        if (r != PISA_OK) return r;
    }
    r = run_select(q, kbar, g, dtype, K, nullptr, mask, s, rbias);
    if (r != PISA_OK) return r;
    if (pooled) {
        // PWT's pooled w as the forward forms it, then the order-3 kernels and the pooled w's
        // gradient into dq and dk
        float* var = (float*)(ws + w.var);
        float* q2 = (float*)(ws + w.q2);
        float* wmat = (float*)(ws + w.wmat);
        float* wsum = (float*)(ws + w.wsum);
        float* wpart = (float*)(ws + w.wpart);
        r = run_wpool(q, k, g, dtype, flags & PISA_FLAG_GATE_W, var, q2, wmat, s);
        if (r != PISA_OK) return r;
        r = run_backward_tc(q, k, v, o, dO, mask, g, 3, flags & PISA_FLAG_GATE_W, lse, (float*)(ws + w.mstat),
                            (float*)(ws + w.dinv), (float*)(ws + w.delta), (float*)(ws + w.lse), dq, dk, dv, s, wmat,
                            wpart);
        if (r != PISA_OK) return r;
        const dim3 grid((unsigned)g.nblk, (unsigned)g.BH);
        const size_t smem = sizeof(float) * g.nblk;
        cudaError_t e = cudaSuccess;
#define PISA_POOLED_BWD(DD, BB)                                                                                   \
    if (g.d == DD && g.B == BB) {                                                                                 \
        pisa::bwdtc::bwd_pooled_dq_kernel<DD, BB><<<grid, 128, smem, s>>>((const bf16*)q, wmat, wpart, var, wsum, \
                                                                         dq, (int)g.L, (int)g.nblk);            \
        e = cudaGetLastError();                                                                                   \
        if (e == cudaSuccess) {                                                                                   \
            pisa::bwdtc::bwd_pooled_dk_kernel<DD, BB><<<grid, 128, 0, s>>>((const bf16*)k, kbar, wsum, q2, dk,    \
                                                                          (int)g.L, (int)g.nblk);               \
            e = cudaGetLastError();                                                                               \
        }                                                                                                         \
    }
        PISA_POOLED_BWD(64, 64)
        PISA_POOLED_BWD(64, 128)
        PISA_POOLED_BWD(128, 64)
        PISA_POOLED_BWD(128, 128)
#undef PISA_POOLED_BWD
        if (e != cudaSuccess) return cuda_fail(e, "pooled-w backward kernels");
        return PISA_OK;
    }
    if (tc_path_available(g, dtype))
        return run_backward_tc(q, k, v, o, dO, mask, g, order, flags & PISA_FLAG_GATE_W, lse, (float*)(ws + w.mstat),
                               (float*)(ws + w.dinv), (float*)(ws + w.delta), (float*)(ws + w.lse), dq, dk, dv, s);
    return run_backward(q, k, v, o, dO, mask, g, dtype, order, flags & PISA_FLAG_GATE_W, (float*)(ws + w.mstat),
                        (float*)(ws + w.dinv), (float*)(ws + w.delta), dq, dk, dv, s);
}

}  // namespace

extern "C" {

pisa_status pisa_attention_backward(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                    int batch, int heads, int L, int d, pisa_dtype dtype, int B, int K, int order,
                                    int flags, float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes,
                                    void* stream) {
    return backward_impl(q, k, v, o, dO, batch, heads, L, d, dtype, B, K, order, flags, nullptr, dq, dk, dv,
                         workspace, ws_bytes, stream);
}

pisa_status pisa_attention_backward_lse(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                        const float* lse, int batch, int heads, int L, int d, pisa_dtype dtype, int B,
                                        int K, int order, int flags, float* dq, float* dk, float* dv,
                                        void* workspace, size_t ws_bytes, void* stream) {
    if (!lse) return fail(PISA_ERR_INVALID_ARG, "pisa_attention_backward_lse: null lse");
    if ((uintptr_t)lse % 4) return fail(PISA_ERR_INVALID_ARG, "pisa_attention_backward_lse: lse must be 4-byte aligned");
    return backward_impl(q, k, v, o, dO, batch, heads, L, d, dtype, B, K, order, flags, lse, dq, dk, dv, workspace,
                         ws_bytes, stream);
}

pisa_status pisa_centroids(const void* k, int batch, int heads, int L, int d, pisa_dtype dtype, int B, float* kbar,
                           void* stream) {
    Dims g;
    pisa_status r = check_dims(batch, heads, L, d, B, 0, dtype, &g);
    if (r != PISA_OK) return r;
    if (!k || !kbar) return fail(PISA_ERR_INVALID_ARG, "pisa_centroids: null k or kbar");
    r = check_align16("pisa_centroids", {k, kbar});
    if (r != PISA_OK) return r;
    return run_centroids(k, kbar, g, dtype, (cudaStream_t)stream);
}

pisa_status pisa_fused_attention(const void* q, const void* k, const void* v, int batch, int heads, int L, int d,
                                 pisa_dtype dtype, int B, int order, int gate_w, pisa_path path,
                                 const uint32_t* mask, const pisa_stats_t* st, void* out, void* stream) {
    Dims g;
    pisa_status r = check_dims(batch, heads, L, d, B, order, dtype, &g);
    if (r != PISA_OK) return r;
    if (!q || !k || !v || !out || !mask) return fail(PISA_ERR_INVALID_ARG, "pisa_fused_attention: null pointer");
    r = check_align16("pisa_fused_attention", {q, k, v, out});
    if (r != PISA_OK) return r;
    if (st) {
        r = check_align16("pisa_fused_attention", {st->kbar, st->vsum, st->hstat, st->cov, st->kaug});
        if (r != PISA_OK) return r;
    }
    // without K, AUTO here takes the token form on the tensor cores, else the statistics path
    if (path == PISA_PATH_AUTO) path = tc_path_available(g, dtype) ? PISA_PATH_RECOMPUTE_TC : PISA_PATH_STATS;
    if (path == PISA_PATH_STATS_TC) {
        if (!stc_path_available(g, dtype, order, false))
            return fail(PISA_ERR_UNSUPPORTED, "statistics-form tensor-core path needs bf16, d and B in {64, 128}, "
                                              "L %% 128 == 0 and order 1");
        if (gate_w & PISA_FLAG_POOLED_W)
            return fail(PISA_ERR_UNSUPPORTED, "pisa_fused_attention: the pooled w needs pisa_attention_ex");
        Dims gs;
        r = check_stats(st, &gs);
        if (r != PISA_OK) return r;
        if (gs.BH != g.BH || gs.L != g.L || gs.d != g.d || gs.B != g.B || st->dtype != dtype)
            return fail(PISA_ERR_INVALID_ARG, "pisa_fused_attention: statistics of another shape");
        if (st->order < 1 || !st->kaug)
            return fail(PISA_ERR_INVALID_ARG, "pisa_fused_attention: the statistics-form tensor-core path needs "
                                              "statistics of order >= 1 with kaug");
        unsigned int* status = device_status_ptr();
        if (!status) return fail(PISA_ERR_CUDA, "cannot resolve the device status word");
        return pisa::run_attn_stc(q, k, v, st->hstat, st->kaug, st->vsum, mask, out, g.BH, (int)g.L, (int)g.d,
                                  (int)g.B, (int)g.nblk, (int)g.words, order, gate_w & PISA_FLAG_GATE_W, nullptr,
                                  status, (cudaStream_t)stream, &g_last_error);
    }
    if (path == PISA_PATH_RECOMPUTE_TC) {
        if (!tc_path_available(g, dtype))
            return fail(PISA_ERR_UNSUPPORTED, "tensor-core path needs bf16, d and B in {64, 128}, L %% 128 == 0");
        unsigned int* status = device_status_ptr();
        if (!status) return fail(PISA_ERR_CUDA, "cannot resolve the device status word");
        if (gate_w & PISA_FLAG_POOLED_W)
            return fail(PISA_ERR_UNSUPPORTED, "pisa_fused_attention: the pooled w needs pisa_attention_ex");
        return pisa::run_attn_tc(q, k, v, mask, out, g.BH, (int)g.L, (int)g.d, (int)g.B, (int)g.nblk,
                                 (int)g.words, order, gate_w & PISA_FLAG_GATE_W, nullptr, status,
                                 (cudaStream_t)stream, &g_last_error);
    }
    if (path != PISA_PATH_STATS) return fail(PISA_ERR_INVALID_ARG, "unknown path %d", (int)path);
    Dims gs;
    r = check_stats(st, &gs);
    if (r != PISA_OK) return r;
    if (gs.BH != g.BH || gs.L != g.L || gs.d != g.d || gs.B != g.B || st->dtype != dtype)
        return fail(PISA_ERR_INVALID_ARG, "pisa_fused_attention: statistics of another shape");
    if (st->order < order) return fail(PISA_ERR_INVALID_ARG, "statistics of order %d for attention of order %d",
                                       st->order, order);
    if (gate_w & PISA_FLAG_POOLED_W)
        return fail(PISA_ERR_UNSUPPORTED, "pisa_fused_attention: the pooled w needs pisa_attention_ex");
    return run_attn_stats(q, k, v, st, mask, out, g, order, gate_w & PISA_FLAG_GATE_W, (cudaStream_t)stream);
}

pisa_status pisa_selftest_wait_timeout(long long limit_cycles, void* stream) {
    if (limit_cycles < 1 || limit_cycles > pisa::kWaitLimitCycles)
        return fail(PISA_ERR_INVALID_ARG, "pisa_selftest_wait_timeout: limit_cycles must be in [1, %lld] (got %lld)",
                    (long long)pisa::kWaitLimitCycles, limit_cycles);
    unsigned int* status = device_status_ptr();
    if (!status) return fail(PISA_ERR_CUDA, "cannot resolve the device status word");
    pisa::wait_timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status, limit_cycles);
    return launch_check("wait_timeout_selftest_kernel");
}

pisa_status pisa_selftest_ex2(const float* x, float* y, long long n, int which, void* stream) {
    if (n < 0) return fail(PISA_ERR_INVALID_ARG, "pisa_selftest_ex2: n must be >= 0 (got %lld)", n);
    if (which != 0 && which != 1) return fail(PISA_ERR_INVALID_ARG, "pisa_selftest_ex2: which must be 0 or 1");
    if (n == 0) return PISA_OK;
    if (!x || !y) return fail(PISA_ERR_INVALID_ARG, "pisa_selftest_ex2: null pointer");
    if ((uintptr_t)x % 4 || (uintptr_t)y % 4)
        return fail(PISA_ERR_INVALID_ARG, "pisa_selftest_ex2: arrays must be 4-byte aligned");
    const long long blocks = (n + 255) / 256;
    pisa::ex2_selftest_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, (cudaStream_t)stream>>>(x, y, n,
                                                                                                       which);
    return launch_check("ex2_selftest_kernel");
}

pisa_status pisa_poll_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int* p = device_status_ptr();
    if (!p) return fail(PISA_ERR_CUDA, "cannot resolve the device status word");
    unsigned int v = 0;
    e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
    const unsigned int zero = 0;
    e = cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status reset)");
    if (v & pisa::kStatusTimeout)
        return fail(PISA_ERR_DEVICE_TIMEOUT, "a device-side wait gave up (status 0x%x)", v);
    if (v) return fail(PISA_ERR_CUDA, "device status 0x%x", v);
    return PISA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of pisa_attention.
//
// pisa_attention asks its caller for device workspace (centroids, selection
// and, on the statistics path, H_j and C_j).  Some callers cannot provide it
// because they may not allocate device memory at all: a plugin inside a host
// application that owns the whole device memory pool and forbids cudaMalloc,
// or a latency-critical loop where cudaMalloc/cudaFree are not allowed
// (cudaFree synchronises the whole device).  For them this entry point takes
// its workspace from a fixed array compiled into the library instead.
//
// The array lives in device memory of every GPU that loads this library, for
// as long as the process runs.  Its name is only a host-side stand-in, so its
// device address is looked up once per device (cudaGetSymbolAddress with that
// device current) and cached.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr size_t kNoallocScratchBytes = (size_t)32 << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[64] = {nullptr};

// Set-up of the current device: resolve the scratch array's device address.
pisa_status noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "pisa_attention_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(PISA_ERR_UNSUPPORTED, "pisa_attention_noalloc: device id %d >= 64", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "pisa_attention_noalloc: cudaGetSymbolAddress");
        if (!p) return fail(PISA_ERR_CUDA, "pisa_attention_noalloc: null scratch address");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return PISA_OK;
}

}  // namespace

extern "C" pisa_status pisa_attention_noalloc(const void* q, const void* k, const void* v, int batch, int heads,
                                              int L, int d, pisa_dtype dtype, int B, int K, int order, void* out,
                                              void* stream) {
    Dims g;
    pisa_status r = check_dims(batch, heads, L, d, B, order, dtype, &g);
    if (r != PISA_OK) return r;
    if (K < 0 || K > g.nblk) return fail(PISA_ERR_INVALID_ARG, "K must be in [0, %ld] (got %d)", g.nblk, K);
    const size_t need = pisa_workspace_bytes(batch, heads, L, d, B, K, order, dtype);
    if (need == 0) return fail(PISA_ERR_INVALID_ARG, "pisa_attention_noalloc: no path for these arguments");
    if (need > kNoallocScratchBytes)
        return fail(PISA_ERR_INVALID_ARG,
                    "pisa_attention_noalloc: this call needs %zu bytes of scratch but the library's built-in "
                    "scratch holds %zu bytes; use pisa_attention with a caller-provided workspace",
                    need, kNoallocScratchBytes);
    void* scratch = nullptr;
    r = noalloc_scratch(&scratch);
    if (r != PISA_OK) return r;
    return pisa_attention_ex(q, k, v, batch, heads, L, d, dtype, B, K, order, 1, PISA_PATH_AUTO, out, scratch,
                             kNoallocScratchBytes, stream);
}

extern "C" size_t pisa_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

// ---------------------------------------------------------------------------
// Host-resident inputs: chunked, double-buffered pisa_attention_ex.
// (batch, head) units are independent, so the heads are cut into chunks and
// chunk c runs on stream c % 2: copy in, attention, copy out.  Copies of one
// chunk overlap the attention of the other on the copy engines.
// ---------------------------------------------------------------------------
namespace {

struct HostSlot {
    char *q, *k, *v, *o, *ws;
};

size_t host_slot_bytes(long chunk, int L, int d, int B, int K, int order, pisa_dtype dtype, pisa_path path) {
    const size_t t = align_up((size_t)chunk * L * d * esize(dtype));
    const size_t ws = pisa_workspace_bytes_ex(1, (int)chunk, L, d, B, K, order, dtype, path);
    if (!ws) return 0;
    return 4 * t + align_up(ws);
}

}  // namespace

extern "C" size_t pisa_attention_host_bytes(int batch, int heads, int L, int d, pisa_dtype dtype, int B, int K,
                                            int order, pisa_path path, int chunk_heads) {
    if (batch <= 0 || heads <= 0 || chunk_heads <= 0) return 0;
    const long BH = (long)batch * heads;
    const long chunk = chunk_heads < BH ? chunk_heads : BH;
    const size_t slot = host_slot_bytes(chunk, L, d, B, K, order, dtype, path);
    return slot ? 2 * slot : 0;
}

extern "C" pisa_status pisa_attention_host(const void* q_host, const void* k_host, const void* v_host,
                                           void* out_host, int batch, int heads, int L, int d, pisa_dtype dtype,
                                           int B, int K, int order, int gate_w, pisa_path path, int chunk_heads,
                                           void* device_buf, size_t device_bytes, void* stream0, void* stream1) {
    Dims g;
    pisa_status r = check_dims(batch, heads, L, d, B, order, dtype, &g);
    if (r != PISA_OK) return r;
    if (!q_host || !k_host || !v_host || !out_host || !device_buf)
        return fail(PISA_ERR_INVALID_ARG, "pisa_attention_host: null pointer");
    if (chunk_heads <= 0) return fail(PISA_ERR_INVALID_ARG, "pisa_attention_host: chunk_heads must be positive");
    if ((uintptr_t)device_buf % kAlign)
        return fail(PISA_ERR_INVALID_ARG, "pisa_attention_host: device_buf must be 256-byte aligned");
    if (path == PISA_PATH_AUTO) path = resolve(g, K, order, dtype);
    const long chunk = chunk_heads < g.BH ? chunk_heads : g.BH;
    const size_t slot = host_slot_bytes(chunk, L, d, B, K, order, dtype, path);
    if (!slot) return fail(PISA_ERR_INVALID_ARG, "pisa_attention_host: no path for these arguments");
    if (device_bytes < 2 * slot)
        return fail(PISA_ERR_INVALID_ARG, "pisa_attention_host: device_buf of %zu bytes, need %zu", device_bytes,
                    2 * slot);
    const size_t t = align_up((size_t)chunk * L * d * esize(dtype));
    HostSlot sl[2];
    for (int i = 0; i < 2; ++i) {
        char* b = (char*)device_buf + i * slot;
        sl[i] = HostSlot{b, b + t, b + 2 * t, b + 3 * t, b + 4 * t};
    }
    cudaStream_t st[2] = {(cudaStream_t)stream0, (cudaStream_t)stream1};
    const size_t head_bytes = (size_t)L * d * esize(dtype);
    int c = 0;
    for (long h0 = 0; h0 < g.BH; h0 += chunk, ++c) {
        const long nh = (g.BH - h0) < chunk ? (g.BH - h0) : chunk;
        const HostSlot& s = sl[c & 1];
        cudaStream_t sm = st[c & 1];
        const size_t off = (size_t)h0 * head_bytes, nb = (size_t)nh * head_bytes;
        cudaError_t e;
        if ((e = cudaMemcpyAsync(s.q, (const char*)q_host + off, nb, cudaMemcpyHostToDevice, sm)) != cudaSuccess ||
            (e = cudaMemcpyAsync(s.k, (const char*)k_host + off, nb, cudaMemcpyHostToDevice, sm)) != cudaSuccess ||
            (e = cudaMemcpyAsync(s.v, (const char*)v_host + off, nb, cudaMemcpyHostToDevice, sm)) != cudaSuccess)
            return cuda_fail(e, "pisa_attention_host: cudaMemcpyAsync (in)");
        r = pisa_attention_ex(s.q, s.k, s.v, 1, (int)nh, L, d, dtype, B, K, order, gate_w, path, s.o, s.ws,
                              slot - 4 * t, sm);
        if (r != PISA_OK) return r;
        if ((e = cudaMemcpyAsync((char*)out_host + off, s.o, nb, cudaMemcpyDeviceToHost, sm)) != cudaSuccess)
            return cuda_fail(e, "pisa_attention_host: cudaMemcpyAsync (out)");
    }
    return PISA_OK;
}
