// Plain CPU oracle for piecewise sparse attention (PISA / PWT).
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
// call this file: only the test-suite, the package smoke check and the CPU
// baseline leg of the benchmark use it.  It shares no code with the CUDA
// library (no headers, helpers or tables) and is deliberately slow: fp64
// arithmetic, one query at a time, loops written in the order the pages state
// the method.  Every floating-point result here is fp64 except the block
// selection, which follows a canonical fp32 procedure (below) so that the GPU
// can reproduce it bit for bit.
//
// Sources (the web pages this method is described on):
//   [blog1] "Sparse Linear Attention" (haoyizhu.site), notation paragraph and
//           sections "Sparse Attention", "Sparse Linear Attention",
//           "Going Further: Adding the Second-Order Term (PWT)".
//   [blog2] "Sparse Linear Attention: When Sparsity Meets Linear Attention (2)",
//           section "Picking Up Where We Left Off" (defines w_{t,j} and H_j).
//   [pisa]  "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
//           Transformers": section 3.1 Eq. 1, section 3.2 "Formulation"
//           (o_t = N_t / D_t and D_t), Figure 3 caption (prepare phase),
//           Appendix C "Notation" (k-bar_j, alpha_{t,j}, delta_{t,j,n}).
//
// Readings taken where the pages are silent:
//   * N_t is not printed in any surviving equation; [blog1] "Sparse Linear
//     Attention" names its three parts (exact, zeroth order, first-order
//     correction with H_j), which gives
//       N_t = sum_{S} sum_n e^{x} v_n + sum_{U} e^{s-bar + w} (vsum_j + H_j q_t).
//   * Selection is per query tile of B rows and scores the tile-mean query
//     against each key centroid ([pisa] Figure 3 caption and section 3.2);
//     ties go to the lower block index.  Eq. 7's softmax is monotone and is
//     dropped; the 1/sqrt(d) is already inside q.
//   * C_j carries 1/B (the second-order expansion of the block mean of
//     e^{y} gives (1/2B) sum_n y_n^2 = 1/2 q^T C_j q).
//   * The PWT gate: w is set to 0 (not clamped) when w > ln B.
//
// Build: g++ -O2 -std=c++17 -fPIC -shared -pthread -ffp-contract=off
// (contraction off so that the fp32 selection rounds every product and sum).

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Canonical fp32 reduction: pairwise tree over a power-of-two count.
// For h = n/2, n/4, ..., 1: a[i] = a[i] + a[i+h] for i < h.  Result a[0].
// Every add is one IEEE fp32 round-to-nearest operation.
// ---------------------------------------------------------------------------
float tree_sum_f32(float* a, long n) {
    for (long h = n / 2; h >= 1; h /= 2) {
        for (long i = 0; i < h; ++i) {
            volatile float s = a[i] + a[i + h];  // volatile: no reassociation
            a[i] = s;
        }
    }
    return a[0];
}

bool is_pow2(long x) { return x > 0 && (x & (x - 1)) == 0; }

// ---------------------------------------------------------------------------
// Reproducible fp32 natural logarithm (for the routing bias, which decides the
// block selection and so must be computed identically by every
// implementation).  Method: x = 2^e m with m in [sqrt(1/2), sqrt(2)); then
// ln m = 2 atanh(s) with s = (m - 1) / (m + 1), |s| <= 0.1716, from the series
// atanh(s) = s + s^3/3 + s^5/5 + s^7/7 + s^9/9 (truncation below 2e-10
// relative); ln x = e ln 2 + ln m.  Every step is one IEEE fp32 operation in a
// fixed order (no FMA contraction).  Defined for finite x > 0 of normal range.
// ---------------------------------------------------------------------------
float ln_f32_canonical(float x) {
    uint32_t bits;
    std::memcpy(&bits, &x, 4);
    int e = (int)((bits >> 23) & 0xffu) - 127;
    uint32_t mb = (bits & 0x007fffffu) | 0x3f800000u;  // m in [1, 2)
    float m;
    std::memcpy(&m, &mb, 4);
    if (m > 0x1.6a09e6p+0f) {  // fp32 sqrt(2)  // fold to [sqrt(1/2), sqrt(2)): halving is exact
        volatile float h = m * 0.5f;
        m = h;
        e += 1;
    }
    volatile float num = m - 1.0f;  // exact (Sterbenz)
    volatile float den = m + 1.0f;
    volatile float sv = num / den;
    const float s = sv;
    volatile float s2 = s * s;
    // Horner in s^2 on the coefficients 1/9, 1/7, 1/5, 1/3, 1 (each fp32 op rounded)
    volatile float t = 0x1.c71c72p-4f * s2;  // fp32 1/9, 1/7, 1/5, 1/3 (round to nearest)
    t = t + 0x1.24924ap-3f;
    t = t * s2;
    t = t + 0x1.99999ap-3f;
    t = t * s2;
    t = t + 0x1.555556p-2f;
    t = t * s2;
    t = t + 1.0f;
    volatile float lnm = t * s;
    lnm = lnm * 2.0f;
    volatile float el = (float)e * 0x1.62e43p-1f;  // fp32 ln 2
    volatile float r = el + lnm;
    return r;
}

// Routing bias of one (bh) for the covariance-aware block selection ([pisa]
// section 3.3 "Covariance-Aware Block Selection": log(M_j + eps) added to the
// centroid score; [blog1] PWT section: log of the norm of H_j).  Canonical fp32:
//   kbar_j[c]  = tree_sum_f32(k[jB..jB+B)[c]) * (1/B)           (the selection's means)
//   dev[n][b]  = k_{j,n}[b] - kbar_j[b]
//   h[a*d + b] = tree_sum_f32 over n of (v_{j,n}[a] * dev[n][b])   (H_j, value channel a)
//   M_j        = sqrt(tree_sum_f32 over a*d+b of h^2)             (Frobenius norm)
//   bias_j     = ln_f32_canonical(M_j + eps)
void route_bias_one(const float* k, const float* v, long L, long d, long B, float eps, float* bias) {
    const long nblk = L / B;
    const float inv_b = 1.0f / (float)B;
    std::vector<float> col(B), kb(d), dev(B * d), prod(B), h(d * d);
    for (long j = 0; j < nblk; ++j) {
        const float* kj = k + j * B * d;
        const float* vj = v + j * B * d;
        for (long c = 0; c < d; ++c) {
            for (long n = 0; n < B; ++n) col[n] = kj[n * d + c];
            volatile float m = tree_sum_f32(col.data(), B) * inv_b;
            kb[c] = m;
        }
        for (long n = 0; n < B; ++n)
            for (long c = 0; c < d; ++c) {
                volatile float x = kj[n * d + c] - kb[c];
                dev[n * d + c] = x;
            }
        for (long a = 0; a < d; ++a)
            for (long b = 0; b < d; ++b) {
                for (long n = 0; n < B; ++n) {
                    volatile float p = vj[n * d + a] * dev[n * d + b];
                    prod[n] = p;
                }
                h[a * d + b] = tree_sum_f32(prod.data(), B);
            }
        for (long e = 0; e < d * d; ++e) {
            volatile float sq = h[e] * h[e];
            h[e] = sq;
        }
        const float m2 = tree_sum_f32(h.data(), d * d);
        volatile float mj = std::sqrt(m2);  // IEEE correctly rounded
        volatile float arg = mj + eps;
        bias[j] = ln_f32_canonical(arg);
    }
}

// Per (bh): fp64 block statistics of the keys and values.
//   kbar_j = (1/B) sum_n k_{j,n}                         ([blog1] notation)
//   vsum_j = sum_n v_{j,n}                               ([pisa] Figure 3)
//   H_j[a][b] = sum_n v_{j,n}[a] (k_{j,n}[b] - kbar_j[b]) ([blog1] "Sparse Linear Attention")
//   C_j[a][b] = (1/B) sum_n (k-kbar)[a] (k-kbar)[b]      ([blog1] PWT section)
void block_stats_one(const float* k, const float* v, long L, long d, long B,
                     double* kbar, double* vsum, double* H, double* C) {
    const long nblk = L / B;
    std::vector<double> dev(B * d);
    for (long j = 0; j < nblk; ++j) {
        const float* kj = k + j * B * d;
        const float* vj = v + j * B * d;
        double* kb = kbar + j * d;
        for (long c = 0; c < d; ++c) {
            double s = 0.0;
            for (long n = 0; n < B; ++n) s += (double)kj[n * d + c];
            kb[c] = s / (double)B;
        }
        if (vsum) {
            double* vs = vsum + j * d;
            for (long c = 0; c < d; ++c) {
                double s = 0.0;
                for (long n = 0; n < B; ++n) s += (double)vj[n * d + c];
                vs[c] = s;
            }
        }
        for (long n = 0; n < B; ++n)
            for (long c = 0; c < d; ++c) dev[n * d + c] = (double)kj[n * d + c] - kb[c];
        if (H) {
            double* Hj = H + j * d * d;
            for (long a = 0; a < d; ++a)
                for (long b = 0; b < d; ++b) {
                    double s = 0.0;
                    for (long n = 0; n < B; ++n) s += (double)vj[n * d + a] * dev[n * d + b];
                    Hj[a * d + b] = s;
                }
        }
        if (C) {
            double* Cj = C + j * d * d;
            for (long a = 0; a < d; ++a)
                for (long b = 0; b < d; ++b) {
                    double s = 0.0;
                    for (long n = 0; n < B; ++n) s += dev[n * d + a] * dev[n * d + b];
                    Cj[a * d + b] = s / (double)B;
                }
        }
    }
}

// Canonical fp32 block selection for one (bh).  For each query tile i:
//   qbar_i[c] = tree_sum_f32(q[iB..iB+B)[c]) * (1/B)      (fp32)
//   kbar_j[c] = tree_sum_f32(k[jB..jB+B)[c]) * (1/B)      (fp32)
//   s_ij      = tree_sum_f32(qbar_i[c] * kbar_j[c] over c) (products rounded)
//   S_i = the K blocks first in the order (s descending, j ascending).
//   with a routing bias (covariance-aware selection): s_ij = s_ij + bias_j (fp32).
void select_one(const float* q, const float* k, long L, long d, long B, long K,
                int32_t* idx, uint32_t* mask, float* scores, const float* bias = nullptr) {
    const long nblk = L / B;
    const long words = (nblk + 31) / 32;
    const float inv_b = 1.0f / (float)B;
    std::vector<float> qbar(nblk * d), kbar(nblk * d), col(B), prod(d), s(nblk);
    for (long j = 0; j < nblk; ++j)
        for (long c = 0; c < d; ++c) {
            for (long n = 0; n < B; ++n) col[n] = k[(j * B + n) * d + c];
            volatile float m = tree_sum_f32(col.data(), B) * inv_b;
            kbar[j * d + c] = m;
        }
    for (long i = 0; i < nblk; ++i)
        for (long c = 0; c < d; ++c) {
            for (long n = 0; n < B; ++n) col[n] = q[(i * B + n) * d + c];
            volatile float m = tree_sum_f32(col.data(), B) * inv_b;
            qbar[i * d + c] = m;
        }
    std::vector<long> order(nblk);
    for (long i = 0; i < nblk; ++i) {
        for (long j = 0; j < nblk; ++j) {
            for (long c = 0; c < d; ++c) {
                volatile float p = qbar[i * d + c] * kbar[j * d + c];
                prod[c] = p;
            }
            s[j] = tree_sum_f32(prod.data(), d);
            if (bias) {
                volatile float sb = s[j] + bias[j];
                s[j] = sb;
            }
            if (scores) scores[i * nblk + j] = s[j];
        }
        for (long j = 0; j < nblk; ++j) order[j] = j;
        std::stable_sort(order.begin(), order.end(), [&](long a, long b) {
            if (s[a] > s[b]) return true;
            if (s[a] < s[b]) return false;
            return a < b;
        });
        uint32_t* mrow = mask ? mask + i * words : nullptr;
        if (mrow) std::memset(mrow, 0, sizeof(uint32_t) * words);
        std::vector<long> chosen(order.begin(), order.begin() + K);
        std::sort(chosen.begin(), chosen.end());
        for (long r = 0; r < K; ++r) {
            if (idx) idx[i * K + r] = (int32_t)chosen[r];
            if (mrow) mrow[chosen[r] / 32] |= (1u << (chosen[r] % 32));
        }
    }
}

// One query row of the statistics form ([pisa] section 3.2 "Formulation",
// [blog1] "Sparse Linear Attention" and PWT section):
//   x_{j,n} = q.k_{j,n}                      j in S (exact)
//   l_j     = q.kbar_j + w_j                  j in U (virtual token logit)
//   w_j     = order 2 ? 1/2 q^T C_j q : 0; with the gate, w_j = 0 when w_j > ln B
//   D = sum_S sum_n e^{x} + sum_U B e^{l}
//   N = sum_S sum_n e^{x} v_n + sum_U e^{l} (vsum_j + [order>=1] H_j q)
//   o = N / D                   (evaluated with the common shift m = max logit)
// With Hbar given, H_j is replaced by the global statistic H-bar (the PISA
// hybrid: first-order term (sum_U e^{l}) H-bar q; [blog1] "Sparse Linear
// Attention", [pisa] section 3.3 and Appendix C, R_t = sum_U alpha (H_j - H-bar)).
void row_stats_form(const float* qrow, const float* k, const float* v, long d, long B,
                    long nblk, const uint8_t* sel, int order, int gate,
                    const double* kbar, const double* vsum, const double* H, const double* C,
                    const double* Hbar, const double* wpool, double* out, double* lse,
                    std::vector<double>& xs, std::vector<double>& ls, std::vector<double>& num) {
    std::vector<double> q(d);
    for (long c = 0; c < d; ++c) q[c] = (double)qrow[c];
    const double ln_b = std::log((double)B);
    double m = -INFINITY;
    for (long j = 0; j < nblk; ++j) {
        if (sel[j]) {
            for (long n = 0; n < B; ++n) {
                const float* kr = k + (j * B + n) * d;
                double x = 0.0;
                for (long c = 0; c < d; ++c) x += q[c] * (double)kr[c];
                xs[j * B + n] = x;
                m = std::max(m, x);
            }
        } else {
            double sb = 0.0;
            for (long c = 0; c < d; ++c) sb += q[c] * kbar[j * d + c];
            double w = 0.0;
            if (order == 2 && wpool) {
                w = wpool[j];  // the tile's pooled diagonal estimate (gate already applied)
            } else if (order == 2) {
                const double* Cj = C + j * d * d;
                for (long a = 0; a < d; ++a) {
                    double t = 0.0;
                    for (long b = 0; b < d; ++b) t += Cj[a * d + b] * q[b];
                    w += q[a] * t;
                }
                w *= 0.5;
                if (gate && w > ln_b) w = 0.0;
            }
            ls[j] = sb + w;
            m = std::max(m, ls[j]);
        }
    }
    double D = 0.0;
    std::fill(num.begin(), num.end(), 0.0);
    for (long j = 0; j < nblk; ++j) {
        if (sel[j]) {
            for (long n = 0; n < B; ++n) {
                const double e = std::exp(xs[j * B + n] - m);
                const float* vr = v + (j * B + n) * d;
                D += e;
                for (long c = 0; c < d; ++c) num[c] += e * (double)vr[c];
            }
        } else {
            const double a = std::exp(ls[j] - m);
            D += (double)B * a;
            const double* vs = vsum + j * d;
            for (long c = 0; c < d; ++c) num[c] += a * vs[c];
            if (order >= 1) {
                // per-block H_j, or the global H-bar of the PISA hybrid
                const double* Hj = Hbar ? Hbar : H + j * d * d;
                for (long r = 0; r < d; ++r) {
                    double t = 0.0;
                    for (long c = 0; c < d; ++c) t += Hj[r * d + c] * q[c];
                    num[r] += a * t;
                }
            }
        }
    }
    for (long c = 0; c < d; ++c) out[c] = num[c] / D;
    if (lse) *lse = m + std::log(D);  // log of the unshifted denominator D_t
}

// The same row without any block statistic: every unselected token keeps the
// first-order weight e^{l_j}(1 + delta_n), delta_n = q.(k_n - kbar_j)
// ([pisa] Appendix C notation; [blog1] "Sparse Linear Attention").  Summing
// these per token must give the statistics form because sum_n delta_n = 0.
void row_brute(const float* qrow, const float* k, const float* v, long d, long B, long nblk,
               const uint8_t* sel, int order, int gate, double* out) {
    std::vector<double> q(d), kb(d), num(d, 0.0);
    for (long c = 0; c < d; ++c) q[c] = (double)qrow[c];
    const double ln_b = std::log((double)B);
    // logits per token for S, per block for U; find the shift
    std::vector<double> xs(nblk * B), ls(nblk), sb(nblk);
    double m = -INFINITY;
    for (long j = 0; j < nblk; ++j) {
        for (long n = 0; n < B; ++n) {
            const float* kr = k + (j * B + n) * d;
            double x = 0.0;
            for (long c = 0; c < d; ++c) x += q[c] * (double)kr[c];
            xs[j * B + n] = x;
        }
        if (sel[j]) {
            for (long n = 0; n < B; ++n) m = std::max(m, xs[j * B + n]);
        } else {
            for (long c = 0; c < d; ++c) {
                double s = 0.0;
                for (long n = 0; n < B; ++n) s += (double)k[(j * B + n) * d + c];
                kb[c] = s / (double)B;
            }
            double s = 0.0;
            for (long c = 0; c < d; ++c) s += q[c] * kb[c];
            sb[j] = s;
            double w = 0.0;
            if (order == 2) {
                // w = (1/2B) sum_n delta_n^2 : the mean of the squared deviation
                for (long n = 0; n < B; ++n) {
                    double dl = 0.0;
                    for (long c = 0; c < d; ++c) dl += q[c] * ((double)k[(j * B + n) * d + c] - kb[c]);
                    w += dl * dl;
                }
                w /= 2.0 * (double)B;
                if (gate && w > ln_b) w = 0.0;
            }
            ls[j] = s + w;
            m = std::max(m, ls[j]);
        }
    }
    double D = 0.0;
    for (long j = 0; j < nblk; ++j) {
        for (long n = 0; n < B; ++n) {
            double wt;
            if (sel[j]) {
                wt = std::exp(xs[j * B + n] - m);
            } else {
                const double dl = (order >= 1) ? xs[j * B + n] - sb[j] : 0.0;
                wt = std::exp(ls[j] - m) * (1.0 + dl);
            }
            D += wt;
            const float* vr = v + (j * B + n) * d;
            for (long c = 0; c < d; ++c) num[c] += wt * (double)vr[c];
        }
    }
    for (long c = 0; c < d; ++c) out[c] = num[c] / D;
}

// Gradients of the method's output for one (bh) (no equations on the pages;
// derived here from the forward above, with the selection held fixed, as the
// PWT blog describes training with the routing detached).  Per query row t,
// with G_n = dO_t . v_n, delta = dO_t . o_t and, for an unselected block j,
// E = e^{l}, u_n = x_n - s-bar, G-bar = (1/B) sum_n G_n:
//   exact key n:       dL/dx_n = e^{x_n} (G_n - delta) / D
//   unselected key m:  dL/dx_m = (E/D) [ (dl/dx_m) (sum_n G_n (1 + c1 u_n) - B delta)
//                                        + c1 (G_m - G-bar) ],
//   c1 = [order >= 1], dl/dx_m = 1/B, plus u_m / B for order 2 when the gate is
//   open (w = (1/2B) sum u^2; the gate decision itself is held fixed);
//   dq_t = sum_n dL/dx_tn k_n,  dk_n = sum_t dL/dx_tn q_t,
//   dv_n = sum_t (weight_tn / D_t) dO_t  (weight = the numerator's e^{x} or E (1 + c1 u_n)).
// Evaluated with the common max shift m (it cancels in weight / D).
// Selection mask and fp64 centroids of one (batch, head), as the forward
// forms them (route_eps > 0: the covariance-aware selection).
void backward_prep(const float* q, const float* k, const float* v, long L, long d, long B, long K,
                   float route_eps, std::vector<uint32_t>& mask, std::vector<double>& kbar) {
    const long nblk = L / B;
    const long words = (nblk + 31) / 32;
    mask.assign(nblk * words, 0u);
    std::vector<float> rbias;
    if (route_eps > 0.0f) {
        rbias.resize(nblk);
        route_bias_one(k, v, L, d, B, route_eps, rbias.data());
    }
    select_one(q, k, L, d, B, K, nullptr, mask.data(), nullptr, rbias.empty() ? nullptr : rbias.data());
    kbar.assign(nblk * d, 0.0);
    for (long j = 0; j < nblk; ++j)
        for (long c = 0; c < d; ++c) {
            double sacc = 0.0;
            for (long n = 0; n < B; ++n) sacc += (double)k[(j * B + n) * d + c];
            kbar[j * d + c] = sacc / (double)B;
        }
}

// Query row t: gx[n] = dL/dx_n over all L keys (x_n = q_t.k_n) and pw[n] =
// wt_n / D, the normalised weight of key n in o_t, with the selection (and
// the gate decision) held fixed.  o_given (null, or [L, d]): the forward output
// the caller holds, as a backward operator of (q, k, v, o, dO) receives it;
// delta = dO_t . o_t then uses its row t instead of the recomputed o_t (the
// only place o enters the gradient).
// wpool (null, or [nblk]): the pooled second-order w of this row's tile per block (PWT's
// diagonal + pooled variant, already gated), which replaces the row's own w; it does not
// depend on the row's logits, so dl/dx_n is 1/B.  dlj (with wpool, [nblk]) receives
// dL/dl_tj = (E/D) inner for the unselected blocks (0 for the selected ones).
void backward_row(const float* q, const float* k, const float* v, const float* dO, const float* o_given, long L,
                  long d, long B, const uint32_t* mask, const double* kbar, int order, int gate, long t, double* gx,
                  double* pw, const double* wpool = nullptr, double* dlj = nullptr) {
    const long nblk = L / B;
    const long words = (nblk + 31) / 32;
    const long i = t / B;
    const float* qt = q + t * d;
    const double ln_b = std::log((double)B);
    const int c1 = order >= 1 ? 1 : 0;
    std::vector<double> x(L), wt(L), lj(nblk), sbj(nblk), o(d, 0.0), G(L);
    std::vector<char> open(nblk);
    for (long n = 0; n < L; ++n) {
        double sacc = 0.0;
        for (long c = 0; c < d; ++c) sacc += (double)qt[c] * (double)k[n * d + c];
        x[n] = sacc;
    }
    // forward: block logits and the common shift
    double m = -INFINITY;
    for (long j = 0; j < nblk; ++j) {
        const bool sel = (mask[i * words + j / 32] >> (j % 32)) & 1u;
        if (sel) {
            for (long n = j * B; n < (j + 1) * B; ++n) m = std::max(m, x[n]);
            continue;
        }
        double sb = 0.0;
        for (long c = 0; c < d; ++c) sb += (double)qt[c] * kbar[j * d + c];
        double w = 0.0;
        if (order == 2 && wpool) {
            w = wpool[j];
            open[j] = 0;  // no per-row dependence of w on the logits
        } else {
            if (order == 2) {
                for (long n = j * B; n < (j + 1) * B; ++n) w += (x[n] - sb) * (x[n] - sb);
                w /= 2.0 * (double)B;
            }
            open[j] = !(gate && w > ln_b);
            if (!open[j]) w = 0.0;
        }
        sbj[j] = sb;
        lj[j] = sb + w;
        m = std::max(m, lj[j]);
    }
    double D = 0.0;
    for (long j = 0; j < nblk; ++j) {
        const bool sel = (mask[i * words + j / 32] >> (j % 32)) & 1u;
        for (long n = j * B; n < (j + 1) * B; ++n) {
            wt[n] = sel ? std::exp(x[n] - m) : std::exp(lj[j] - m) * (1.0 + c1 * (x[n] - sbj[j]));
            for (long c = 0; c < d; ++c) o[c] += wt[n] * (double)v[n * d + c];
        }
        D += sel ? 0.0 : (double)B * std::exp(lj[j] - m);
        if (sel)
            for (long n = j * B; n < (j + 1) * B; ++n) D += wt[n];
    }
    for (long c = 0; c < d; ++c) o[c] /= D;
    const float* dOt = dO + t * d;
    double delta = 0.0;
    if (o_given)
        for (long c = 0; c < d; ++c) delta += (double)dOt[c] * (double)o_given[t * d + c];
    else
        for (long c = 0; c < d; ++c) delta += (double)dOt[c] * o[c];
    for (long n = 0; n < L; ++n) {
        double g = 0.0;
        for (long c = 0; c < d; ++c) g += (double)dOt[c] * (double)v[n * d + c];
        G[n] = g;
        pw[n] = wt[n] / D;
    }
    // dL/dx
    for (long j = 0; j < nblk; ++j) {
        const bool sel = (mask[i * words + j / 32] >> (j % 32)) & 1u;
        if (sel) {
            for (long n = j * B; n < (j + 1) * B; ++n) gx[n] = wt[n] * (G[n] - delta) / D;
            if (dlj) dlj[j] = 0.0;
            continue;
        }
        const double E = std::exp(lj[j] - m);
        double sg = 0.0, gbar = 0.0;
        for (long n = j * B; n < (j + 1) * B; ++n) {
            sg += G[n] * (1.0 + c1 * (x[n] - sbj[j]));
            gbar += G[n];
        }
        gbar /= (double)B;
        const double inner = sg - (double)B * delta;
        if (dlj) dlj[j] = (E / D) * inner;
        for (long n = j * B; n < (j + 1) * B; ++n) {
            double dl = 1.0 / (double)B;
            if (order == 2 && open[j]) dl += (x[n] - sbj[j]) / (double)B;
            gx[n] = (E / D) * (dl * inner + c1 * (G[n] - gbar));
        }
    }
}

void backward_one(const float* q, const float* k, const float* v, const float* dO, const float* o_given, long L,
                  long d, long B, long K, int order, int gate, int w_pooled, float route_eps, double* dq, double* dk,
                  double* dv) {
    std::vector<uint32_t> mask;
    std::vector<double> kbar, gx(L), pw(L);
    backward_prep(q, k, v, L, d, B, K, route_eps, mask, kbar);
    const long nblk = L / B;
    const bool pooled = order == 2 && w_pooled;
    // PWT's pooled w (the forward's definition): w_ij = 1/2 sum_c q2_ic sigma2_jc, with
    // q2_ic the tile mean of q_c^2 and sigma2_jc = C_j[c][c] the block's channel variance,
    // gated at ln B.  It is shared by the tile's rows, so its gradient gathers
    // W_ij = sum_{t in tile i} dL/dl_tj over them, then reaches q through q2 and k through
    // sigma2:  dq_mc += W_ij sigma2_jc q_mc / B,  dk_nc += W_ij q2_ic (k_nc - kbar_jc) / B.
    std::vector<double> sig2, q2(d), wp(nblk), dlj(nblk), W(nblk);
    std::vector<char> keep(nblk);
    if (pooled) {
        sig2.assign(nblk * d, 0.0);
        for (long j = 0; j < nblk; ++j)
            for (long c = 0; c < d; ++c) {
                double s2 = 0.0;
                for (long n = j * B; n < (j + 1) * B; ++n) {
                    const double u = (double)k[n * d + c] - kbar[j * d + c];
                    s2 += u * u;
                }
                sig2[j * d + c] = s2 / (double)B;
            }
    }
    const double ln_b = std::log((double)B);
    for (long i = 0; i < nblk; ++i) {
        if (pooled) {
            std::fill(q2.begin(), q2.end(), 0.0);
            for (long m = i * B; m < (i + 1) * B; ++m)
                for (long c = 0; c < d; ++c) q2[c] += (double)q[m * d + c] * (double)q[m * d + c];
            for (long c = 0; c < d; ++c) q2[c] /= (double)B;
            for (long j = 0; j < nblk; ++j) {
                double w = 0.0;
                for (long c = 0; c < d; ++c) w += q2[c] * sig2[j * d + c];
                w *= 0.5;
                keep[j] = !(gate && w > ln_b);
                wp[j] = keep[j] ? w : 0.0;
                W[j] = 0.0;
            }
        }
        for (long t = i * B; t < (i + 1) * B; ++t) {
            backward_row(q, k, v, dO, o_given, L, d, B, mask.data(), kbar.data(), order, gate, t, gx.data(),
                         pw.data(), pooled ? wp.data() : nullptr, pooled ? dlj.data() : nullptr);
            const float* qt = q + t * d;
            const float* dOt = dO + t * d;
            for (long n = 0; n < L; ++n) {
                for (long c = 0; c < d; ++c) {
                    dq[t * d + c] += gx[n] * (double)k[n * d + c];
                    dk[n * d + c] += gx[n] * (double)qt[c];
                    dv[n * d + c] += pw[n] * (double)dOt[c];
                }
            }
            if (pooled)
                for (long j = 0; j < nblk; ++j)
                    if (keep[j]) W[j] += dlj[j];
        }
        if (pooled) {
            for (long j = 0; j < nblk; ++j) {
                if (!keep[j] || W[j] == 0.0) continue;
                for (long m = i * B; m < (i + 1) * B; ++m)
                    for (long c = 0; c < d; ++c) dq[m * d + c] += W[j] * sig2[j * d + c] * (double)q[m * d + c] / (double)B;
                for (long n = j * B; n < (j + 1) * B; ++n)
                    for (long c = 0; c < d; ++c)
                        dk[n * d + c] += W[j] * q2[c] * ((double)k[n * d + c] - kbar[j * d + c]) / (double)B;
            }
        }
    }
}

template <class F>
void parallel_for(long n, int nthreads, F&& fn) {
    if (nthreads <= 1 || n <= 1) {
        for (long i = 0; i < n; ++i) fn(i);
        return;
    }
    std::atomic<long> next(0);
    std::vector<std::thread> pool;
    const int nt = (int)std::min<long>(nthreads, n);
    for (int t = 0; t < nt; ++t)
        pool.emplace_back([&]() {
            for (;;) {
                long i = next.fetch_add(1);
                if (i >= n) break;
                fn(i);
            }
        });
    for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// Returns 0 on success, -1 on a shape the oracle does not define.
int oracle_block_stats(const float* k, const float* v, long BH, long L, long d, long B,
                       double* kbar, double* vsum, double* H, double* C, int nthreads) {
    if (B <= 0 || L % B) return -1;
    const long nblk = L / B;
    parallel_for(BH, nthreads, [&](long bh) {
        block_stats_one(k + bh * L * d, v + bh * L * d, L, d, B, kbar + bh * nblk * d,
                        vsum ? vsum + bh * nblk * d : nullptr,
                        H ? H + bh * nblk * d * d : nullptr,
                        C ? C + bh * nblk * d * d : nullptr);
    });
    return 0;
}

// Canonical fp32 centroids (the means the selection uses): [BH, nblk, d].
int oracle_centroids_f32(const float* k, long BH, long L, long d, long B, float* kbar, int nthreads) {
    if (!is_pow2(B) || L % B) return -1;
    const long nblk = L / B;
    parallel_for(BH, nthreads, [&](long bh) {
        std::vector<float> col(B);
        const float inv_b = 1.0f / (float)B;
        for (long j = 0; j < nblk; ++j)
            for (long c = 0; c < d; ++c) {
                for (long n = 0; n < B; ++n) col[n] = k[(bh * L + j * B + n) * d + c];
                volatile float m = tree_sum_f32(col.data(), B) * inv_b;
                kbar[(bh * nblk + j) * d + c] = m;
            }
    });
    return 0;
}

// Canonical fp32 routing bias ln(||H_j||_F + eps): [BH, nblk].
int oracle_route_bias(const float* k, const float* v, long BH, long L, long d, long B, float eps,
                      float* bias, int nthreads) {
    if (!is_pow2(B) || !is_pow2(d) || L % B || !(eps > 0.0f)) return -1;
    const long nblk = L / B;
    parallel_for(BH, nthreads, [&](long bh) {
        route_bias_one(k + bh * L * d, v + bh * L * d, L, d, B, eps, bias + bh * nblk);
    });
    return 0;
}

// The reproducible fp32 logarithm, element-wise (for its pins).
int oracle_ln_f32(const float* x, long n, float* out) {
    for (long i = 0; i < n; ++i) out[i] = ln_f32_canonical(x[i]);
    return 0;
}

// bias: null for the plain centroid score, else [BH, nblk] added to every score.
int oracle_select(const float* q, const float* k, long BH, long L, long d, long B, long K,
                  int32_t* idx, uint32_t* mask, float* scores, const float* bias, int nthreads) {
    if (!is_pow2(B) || !is_pow2(d) || L % B) return -1;
    const long nblk = L / B;
    if (K < 0 || K > nblk) return -1;
    const long words = (nblk + 31) / 32;
    parallel_for(BH, nthreads, [&](long bh) {
        select_one(q + bh * L * d, k + bh * L * d, L, d, B, K,
                   idx ? idx + bh * nblk * K : nullptr, mask ? mask + bh * nblk * words : nullptr,
                   scores ? scores + bh * nblk * nblk : nullptr, bias ? bias + bh * nblk : nullptr);
    });
    return 0;
}

// Statistics-form output for a list of query tiles.  tiles[2*r] = bh,
// tiles[2*r+1] = tile index i; out receives [ntiles, B, d] fp64 rows and, when
// lse is not null, lse receives [ntiles, B] values log(D_t) (unshifted).
// The selection (canonical fp32) is recomputed here from q and k.
static int pisa_attention_impl(const float* q, const float* k, const float* v, long BH, long L,
                               long d, long B, long K, int order, int gate, int global_h,
                               int w_pooled, float route_eps, const int64_t* tiles, long ntiles,
                               double* out, double* lse, int nthreads) {
    if (!is_pow2(B) || !is_pow2(d) || L % B || order < 0 || order > 2) return -1;
    const long nblk = L / B;
    if (K < 0 || K > nblk) return -1;
    // statistics and selection for every bh that appears in the tile list
    std::vector<char> need(BH, 0);
    for (long r = 0; r < ntiles; ++r) {
        if (tiles[2 * r] < 0 || tiles[2 * r] >= BH || tiles[2 * r + 1] < 0 || tiles[2 * r + 1] >= nblk)
            return -1;
        need[tiles[2 * r]] = 1;
    }
    std::vector<long> bhs;
    for (long bh = 0; bh < BH; ++bh)
        if (need[bh]) bhs.push_back(bh);
    const long words = (nblk + 31) / 32;
    std::vector<std::vector<double>> kbar(BH), vsum(BH), H(BH), C(BH), Hbar(BH);
    std::vector<std::vector<uint32_t>> mask(BH);
    parallel_for((long)bhs.size(), nthreads, [&](long r) {
        const long bh = bhs[r];
        kbar[bh].assign(nblk * d, 0.0);
        vsum[bh].assign(nblk * d, 0.0);
        H[bh].assign(order >= 1 ? nblk * d * d : 0, 0.0);
        C[bh].assign(order == 2 ? nblk * d * d : 0, 0.0);
        block_stats_one(k + bh * L * d, v + bh * L * d, L, d, B, kbar[bh].data(), vsum[bh].data(),
                        order >= 1 ? H[bh].data() : nullptr, order == 2 ? C[bh].data() : nullptr);
        mask[bh].assign(nblk * words, 0u);
        std::vector<float> rbias;
        if (route_eps > 0.0f) {  // covariance-aware selection
            rbias.assign(nblk, 0.0f);
            route_bias_one(k + bh * L * d, v + bh * L * d, L, d, B, route_eps, rbias.data());
        }
        select_one(q + bh * L * d, k + bh * L * d, L, d, B, K, nullptr, mask[bh].data(), nullptr,
                   rbias.empty() ? nullptr : rbias.data());
        if (global_h && order >= 1) {
            // H-bar = (B / L) sum over all blocks of H_j  ([blog1] "Sparse Linear Attention")
            Hbar[bh].assign(d * d, 0.0);
            for (long j = 0; j < nblk; ++j)
                for (long e = 0; e < d * d; ++e) Hbar[bh][e] += H[bh][j * d * d + e];
            for (long e = 0; e < d * d; ++e) Hbar[bh][e] *= (double)B / (double)L;
        }
    });
    parallel_for(ntiles, nthreads, [&](long r) {
        const long bh = tiles[2 * r], i = tiles[2 * r + 1];
        std::vector<uint8_t> sel(nblk);
        for (long j = 0; j < nblk; ++j) sel[j] = (mask[bh][i * words + j / 32] >> (j % 32)) & 1u;
        std::vector<double> xs(nblk * B), ls(nblk), num(d);
        // PWT's cheap w ([blog1] PWT section): the diagonal of C_j (the within-block
        // variance of each channel) weighted by the tile mean of q^2 (square first,
        // then average), one value per (tile, block), gated at ln B.
        std::vector<double> wpool;
        if (order == 2 && w_pooled) {
            std::vector<double> q2(d, 0.0);
            for (long m = 0; m < B; ++m)
                for (long c = 0; c < d; ++c) {
                    const double x = (double)q[(bh * L + i * B + m) * d + c];
                    q2[c] += x * x;
                }
            for (long c = 0; c < d; ++c) q2[c] /= (double)B;
            wpool.assign(nblk, 0.0);
            const double ln_b = std::log((double)B);
            for (long j = 0; j < nblk; ++j) {
                double w = 0.0;
                for (long c = 0; c < d; ++c) w += q2[c] * C[bh][j * d * d + c * d + c];
                w *= 0.5;
                wpool[j] = (gate && w > ln_b) ? 0.0 : w;
            }
        }
        for (long m = 0; m < B; ++m) {
            const long t = i * B + m;
            row_stats_form(q + (bh * L + t) * d, k + bh * L * d, v + bh * L * d, d, B, nblk,
                           sel.data(), order, gate, kbar[bh].data(), vsum[bh].data(),
                           H[bh].data(), C[bh].data(),
                           (global_h && order >= 1) ? Hbar[bh].data() : nullptr,
                           wpool.empty() ? nullptr : wpool.data(), out + (r * B + m) * d,
                           lse ? lse + r * B + m : nullptr, xs, ls, num);
        }
    });
    return 0;
}

int oracle_pisa_attention(const float* q, const float* k, const float* v, long BH, long L,
                          long d, long B, long K, int order, int gate, const int64_t* tiles,
                          long ntiles, double* out, double* lse, int nthreads) {
    return pisa_attention_impl(q, k, v, BH, L, d, B, K, order, gate, 0, 0, 0.0f, tiles, ntiles, out,
                               lse, nthreads);
}

// General form: global_h selects the PISA hybrid's H-bar, w_pooled PWT's
// diagonal + pooled second-order correction (order 2), route_eps > 0 the
// covariance-aware selection with bias ln(||H_j||_F + route_eps).
int oracle_pisa_attention_ex(const float* q, const float* k, const float* v, long BH, long L,
                             long d, long B, long K, int order, int gate, int global_h, int w_pooled,
                             float route_eps, const int64_t* tiles, long ntiles, double* out,
                             double* lse, int nthreads) {
    return pisa_attention_impl(q, k, v, BH, L, d, B, K, order, gate, global_h, w_pooled, route_eps,
                               tiles, ntiles, out, lse, nthreads);
}

// The PISA hybrid: as oracle_pisa_attention with every H_j replaced by the
// global H-bar = (B/L) sum_j H_j of the (batch, head).
int oracle_pisa_hybrid(const float* q, const float* k, const float* v, long BH, long L, long d,
                       long B, long K, int order, int gate, const int64_t* tiles, long ntiles,
                       double* out, double* lse, int nthreads) {
    return pisa_attention_impl(q, k, v, BH, L, d, B, K, order, gate, 1, 0, 0.0f, tiles, ntiles, out,
                               lse, nthreads);
}

// Token-wise form (no block statistics), same selection; full output [BH, L, d].
int oracle_pisa_bruteforce(const float* q, const float* k, const float* v, long BH, long L,
                           long d, long B, long K, int order, int gate, double* out,
                           int nthreads) {
    if (!is_pow2(B) || !is_pow2(d) || L % B || order < 0 || order > 2) return -1;
    const long nblk = L / B;
    if (K < 0 || K > nblk) return -1;
    const long words = (nblk + 31) / 32;
    parallel_for(BH, nthreads, [&](long bh) {
        std::vector<uint32_t> mask(nblk * words);
        select_one(q + bh * L * d, k + bh * L * d, L, d, B, K, nullptr, mask.data(), nullptr);
        std::vector<uint8_t> sel(nblk);
        for (long i = 0; i < nblk; ++i) {
            for (long j = 0; j < nblk; ++j) sel[j] = (mask[i * words + j / 32] >> (j % 32)) & 1u;
            for (long m = 0; m < B; ++m) {
                const long t = i * B + m;
                row_brute(q + (bh * L + t) * d, k + bh * L * d, v + bh * L * d, d, B, nblk,
                          sel.data(), order, gate, out + (bh * L + t) * d);
            }
        }
    });
    return 0;
}

// Gradients (dq, dk, dv) [BH, L, d] fp64 of sum_t dO_t . o_t for the method's
// output o (pisa_attention's), selection held fixed.  Zero-initialised here.
// o_given: null (delta from the recomputed fp64 o) or [BH, L, d], the forward
// output the caller holds (delta = dO_t . o_given_t).  w_pooled (order 2): the
// gradient of PWT's diagonal + pooled w, the gate decisions held fixed.
int oracle_pisa_backward(const float* q, const float* k, const float* v, const float* dO, const float* o_given,
                         long BH, long L, long d, long B, long K, int order, int gate, int w_pooled, float route_eps,
                         double* dq, double* dk, double* dv, int nthreads) {
    if (!is_pow2(B) || !is_pow2(d) || L % B || order < 0 || order > 2) return -1;
    if (K < 0 || K > L / B) return -1;
    std::fill(dq, dq + BH * L * d, 0.0);
    std::fill(dk, dk + BH * L * d, 0.0);
    std::fill(dv, dv + BH * L * d, 0.0);
    parallel_for(BH, nthreads, [&](long bh) {
        const long o = bh * L * d;
        backward_one(q + o, k + o, v + o, dO + o, o_given ? o_given + o : nullptr, L, d, B, K, order, gate, w_pooled,
                     route_eps, dq + o, dk + o, dv + o);
    });
    return 0;
}

// dq of a list of query rows: rows[2*r] = bh, rows[2*r+1] = t; dq_rows
// receives [nrows, d] fp64 (the rows of oracle_pisa_backward's dq).
int oracle_pisa_backward_dq_rows(const float* q, const float* k, const float* v, const float* dO,
                                 const float* o_given, long BH, long L, long d, long B, long K, int order, int gate,
                                 float route_eps, const int64_t* rows, long nrows, double* dq_rows, int nthreads) {
    if (!is_pow2(B) || !is_pow2(d) || L % B || order < 0 || order > 2) return -1;
    if (K < 0 || K > L / B) return -1;
    for (long r = 0; r < nrows; ++r)
        if (rows[2 * r] < 0 || rows[2 * r] >= BH || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= L) return -1;
    std::vector<std::vector<uint32_t>> mask(BH);
    std::vector<std::vector<double>> kbar(BH);
    std::vector<char> used(BH, 0);
    for (long r = 0; r < nrows; ++r) used[rows[2 * r]] = 1;
    parallel_for(BH, nthreads, [&](long bh) {
        if (used[bh])
            backward_prep(q + bh * L * d, k + bh * L * d, v + bh * L * d, L, d, B, K, route_eps, mask[bh], kbar[bh]);
    });
    parallel_for(nrows, nthreads, [&](long r) {
        const long bh = rows[2 * r], t = rows[2 * r + 1];
        const long o = bh * L * d;
        std::vector<double> gx(L), pw(L);
        backward_row(q + o, k + o, v + o, dO + o, o_given ? o_given + o : nullptr, L, d, B, mask[bh].data(),
                     kbar[bh].data(), order, gate, t, gx.data(), pw.data());
        for (long c = 0; c < d; ++c) {
            double acc = 0.0;
            for (long n = 0; n < L; ++n) acc += gx[n] * (double)k[o + n * d + c];
            dq_rows[r * d + c] = acc;
        }
    });
    return 0;
}

// Dense softmax attention o_t = sum_i softmax(q_t.k_i) v_i ([pisa] Eq. 1), fp64.
int oracle_dense_attention(const float* q, const float* k, const float* v, long BH, long L,
                           long d, double* out, int nthreads) {
    parallel_for(BH * L, nthreads, [&](long r) {
        const long bh = r / L;
        const float* qr = q + r * d;
        const float* kh = k + bh * L * d;
        const float* vh = v + bh * L * d;
        std::vector<double> x(L), num(d, 0.0);
        double m = -INFINITY;
        for (long i = 0; i < L; ++i) {
            double s = 0.0;
            for (long c = 0; c < d; ++c) s += (double)qr[c] * (double)kh[i * d + c];
            x[i] = s;
            m = std::max(m, s);
        }
        double D = 0.0;
        for (long i = 0; i < L; ++i) {
            const double e = std::exp(x[i] - m);
            D += e;
            for (long c = 0; c < d; ++c) num[c] += e * (double)vh[i * d + c];
        }
        for (long c = 0; c < d; ++c) out[r * d + c] = num[c] / D;
    });
    return 0;
}

}  // extern "C"
