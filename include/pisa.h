/*
 * pisa.h -- C ABI of the B200 (sm_100a) piecewise sparse attention library.
 *
 * The operation (PISA / PWT piecewise sparse attention):
 *   Keys and values of each (batch, head) are cut in order into blocks of B
 *   tokens.  Query tile i (rows iB .. iB+B-1) keeps the K key blocks whose
 *   centroid scores highest against the tile's mean query (S_i) and gets exact
 *   softmax attention on them; every other block j (U_i) is replaced by its
 *   Taylor expansion around the key centroid kbar_j.  Both parts share one
 *   softmax max and one denominator:
 *     D_t = sum_{j in S_i} sum_n e^{q_t.k_{j,n}} + sum_{j in U_i} B e^{l_tj}
 *     N_t = sum_{j in S_i} sum_n e^{q_t.k_{j,n}} v_{j,n}
 *         + sum_{j in U_i} e^{l_tj} (vsum_j + [order>=1] H_j q_t)
 *     o_t = N_t / D_t,   l_tj = q_t.kbar_j + w_tj,
 *     w_tj = [order==2] 1/2 q_t^T C_j q_t  (set to 0 when it exceeds ln B and
 *            the gate is on).
 *   Definitions: PISA paper ("PISA: Piecewise Sparse Attention Is Wiser for
 *   Efficient Diffusion Transformers"), section 3.2 "Formulation" (o_t, D_t),
 *   Figure 3 caption and section 3.4 (prepare phase, phases 1-2), Appendix C
 *   "Notation" (kbar_j, alpha_tj, delta_tjn); "Sparse Linear Attention" blog,
 *   sections "Sparse Linear Attention" (virtual token, H_j) and "Going Further:
 *   Adding the Second-Order Term (PWT)" (w_tj, C_j, the ln B gate).
 *   The softmax scale is folded into q: callers pass q already multiplied by
 *   1/sqrt(d) (PISA paper section 3.1, Eq. 1; blog notation paragraph).
 *
 * Conventions for every entry point:
 *   - Tensors are row-major [batch*heads, L, d] ("BHLD" with batch and heads
 *     folded), contiguous, element type given by pisa_dtype.
 *   - Every pointer argument is device memory owned by the caller unless a
 *     comment says otherwise.  The library allocates no memory (except the
 *     variant documented at its declaration) and keeps no state other than one
 *     device status word per device.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued asynchronously on it; no call
 *     synchronises the host, except pisa_poll_device_status.
 *   - Supported on the GPU path: d in {64, 128}, B in {64, 128}, L % B == 0,
 *     0 <= K <= L/B, order in {0, 1, 2}, L/B <= 4096.  Other shapes return
 *     PISA_ERR_UNSUPPORTED (valid but not implemented) or
 *     PISA_ERR_INVALID_ARG (meaningless).
 *   - Device arrays (inputs, outputs, statistics) must be 16-byte aligned, as
 *     contiguous allocations are; PISA_ERR_INVALID_ARG otherwise.
 *   - Non-finite inputs give undefined (but memory-safe) results.
 *   - On a non-OK status, pisa_last_error() returns a message for the calling
 *     thread.  Argument errors are detected before anything is enqueued.
 */
#ifndef PISA_H_
#define PISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PISA_OK = 0,
    PISA_ERR_INVALID_ARG = 1,    /* null pointer, bad shape, workspace too small */
    PISA_ERR_UNSUPPORTED = 2,    /* valid but not implemented on this path */
    PISA_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed */
    PISA_ERR_DEVICE_TIMEOUT = 4  /* a bounded device-side wait gave up */
} pisa_status;

typedef enum { PISA_F32 = 0, PISA_BF16 = 1 } pisa_dtype;

/* Which formulation pisa_attention_ex evaluates the unselected blocks with.
 *   PISA_PATH_AUTO          : on the tensor cores (bf16, d and B in {64, 128},
 *                             L % 128 == 0) the one of PISA_PATH_RECOMPUTE_TC
 *                             and PISA_PATH_STATS_TC that executes fewer FLOPs
 *                             (STATS_TC only for order 1; see below), else
 *                             PISA_PATH_STATS.
 *   PISA_PATH_STATS         : statistics form: uses kbar_j, vsum_j, H_j, C_j
 *                             from pisa_stats (CUDA cores, fp32 accumulation).
 *   PISA_PATH_RECOMPUTE_TC  : token form on tcgen05 tensor cores: the
 *                             unselected block's first-order numerator
 *                             e^{l}(vsum_j + H_j q) is evaluated as
 *                             sum_n e^{l}(1 + q.(k_n - kbar_j)) v_n, which is
 *                             the same quantity; w is taken from the same
 *                             logits.  bf16 only, L % 128 == 0.  Executes
 *                             4 L^2 d FLOPs per (batch, head).
 *   PISA_PATH_STATS_TC      : statistics form on tcgen05 tensor cores: blocks
 *                             selected by any query tile of a 256-row CTA run
 *                             in the token form above; every other block's
 *                             term is the contraction H_j q_t (one MMA per
 *                             128 rows and block, with q_t . kbar_j from the
 *                             same MMA).  bf16, L % 128 == 0, order 1 (order 2
 *                             only with PISA_FLAG_POOLED_W).  With U the
 *                             blocks selected by the CTA's tiles, it executes
 *                             per 256 rows 256 (4 d 128 ceil(U / (128/B))
 *                             + 2 d (g d + 16) ceil((L/B - U) / g)) FLOPs,
 *                             g = 2 for d = 64 and 1 for d = 128: fewer than
 *                             the token form when d <= B.  AUTO takes it when
 *                             that count, with U at its bound
 *                             min(L/B, (256/B) K), is below 4 L d per row. */
typedef enum {
    PISA_PATH_AUTO = 0,
    PISA_PATH_STATS = 1,
    PISA_PATH_RECOMPUTE_TC = 2,
    PISA_PATH_HYBRID_TC = 3,
    PISA_PATH_STATS_TC = 4
} pisa_path;
/* PISA_PATH_HYBRID_TC is another method, requested explicitly (AUTO never
 * picks it): the PISA paper's hybrid, where every H_j of the first-order term
 * is replaced by the global statistic H-bar = (B/L) sum_j H_j of the (batch,
 * head), so the numerator's first-order part is (sum_{j in U_i} e^{l_tj})
 * H-bar q_t (PISA paper section 3.3 and Figure 3, phase 3; H-bar as in the
 * "Sparse Linear Attention" blog).  Unselected blocks cost one virtual token
 * each instead of their tokens.  bf16, L % 128 == 0; order 2 only with the
 * pooled w (PISA_FLAG_POOLED_W). */

/* Block statistics of one call (all device pointers, caller-owned).
 *   kbar  [BH, nblk, d] fp32 : centroid, canonical fp32 mean (see pisa_select)
 *   vsum  [BH, nblk, d] fp32 : sum_n v_{j,n}
 *   hstat [BH, nblk, d, d]   : H_j[a][b] = sum_n v_{j,n}[a] (k_{j,n}[b] - kbar_j[b])
 *                              (row = value channel), element type = dtype
 *   cov   [BH, nblk, d, d]   : C_j = (1/B) sum_n (k-kbar)(k-kbar)^T, element
 *                              type = dtype; NULL unless order == 2.
 *   kaug  [BH, nblk, 8, d] bf16 : the centroid split for the tensor cores:
 *                              row 0 = bf16(kbar_j) (round to nearest), row 1 =
 *                              bf16(kbar_j - row 0), rows 2-7 zero; NULL unless
 *                              dtype == PISA_BF16 and order >= 1 (read by
 *                              PISA_PATH_STATS_TC).
 * hstat is NULL when order == 0.  Fill with pisa_stats_bind. */
typedef struct {
    int batch, heads, L, d, B, nblk, order;
    pisa_dtype dtype;
    float* kbar;
    float* vsum;
    void* hstat;
    void* cov;
    void* kaug;
} pisa_stats_t;

/* Bytes of device memory pisa_stats_bind needs for these dimensions
 * (each array 256-byte aligned).  Returns 0 for invalid dimensions. */
size_t pisa_stats_bytes(int batch, int heads, int L, int d, int B, int order, pisa_dtype dtype);

/* Lay out a pisa_stats_t inside caller memory `buf` of `bytes` bytes
 * (buf 256-byte aligned).  No device work.  Errors: INVALID_ARG for a null
 * st/buf, a too-small buffer or invalid dimensions. */
pisa_status pisa_stats_bind(pisa_stats_t* st, void* buf, size_t bytes, int batch, int heads,
                            int L, int d, int B, int order, pisa_dtype dtype);

/* Prepare phase (PISA paper section 3.4, Figure 3): one pass over k and v
 * ([BH, L, d], element type st->dtype) writing every array of *st. */
pisa_status pisa_stats(const void* k, const void* v, const pisa_stats_t* st, void* stream);

/* Block selection (PISA paper section 3.2 and Figure 3; MoBA-style scoring,
 * "Sparse Linear Attention" blog section "Sparse Attention").
 * For each query tile i of q ([BH, L, d], type st->dtype), in fp32 with a fixed
 * reduction order so that the result is reproducible bit for bit:
 *   tsum(a[0..n)) : for h = n/2, ..., 1: a[i] = a[i] + a[i+h] (i < h); a[0]
 *   qbar_i[c] = tsum(q rows of the tile, column c) * (1/B)
 *   s_ij      = tsum over c of (qbar_i[c] * st->kbar[j][c])   (rounded products)
 *   S_i       = the K blocks first under (s descending, j ascending).
 * Outputs: idx [BH, nblk, K] int32, each row ascending (may be NULL);
 *          mask [BH, nblk, ceil(nblk/32)] uint32, bit j%32 of word j/32 set iff
 *          j in S_i (may be NULL).  Only st->kbar is read (pisa_stats or
 *          pisa_centroids output); the other arrays of *st may be NULL. */
pisa_status pisa_select(const void* q, const pisa_stats_t* st, int K, int32_t* idx,
                        uint32_t* mask, void* stream);

/* Covariance-aware block selection (PISA paper, section 3.3 "Covariance-Aware
 * Block Selection": the log of a block norm plus eps is added to the centroid
 * score; "Sparse Linear Attention" blog, PWT section: route by the score plus
 * the log of the norm of H_j).  As pisa_select with every score s_ij replaced
 * by s_ij + bias[bh][j] (one fp32 add, round to nearest) before the top-K.
 * bias: [BH, nblk] fp32 device array (pisa_route_bias output), or NULL for
 * exactly pisa_select. */
pisa_status pisa_select_biased(const void* q, const pisa_stats_t* st, int K, const float* bias,
                               int32_t* idx, uint32_t* mask, void* stream);

/* The score table of the selection: scores [BH, nblk, nblk] fp32 (row = query
 * tile i, column = block j) holding s_ij exactly as pisa_select (bias NULL) or
 * pisa_select_biased computes it before the top-K.  For inspection and tests. */
pisa_status pisa_select_scores(const void* q, const pisa_stats_t* st, const float* bias, float* scores,
                               void* stream);

/* Routing bias bias[bh][j] = ln(||H_j||_F + eps) of every key block, from k and
 * v ([BH, L, d], `dtype`) and the canonical centroids kbar ([BH, nblk, d] fp32,
 * pisa_centroids or pisa_stats output).  It decides a selection, so it is
 * computed in a fixed fp32 procedure that reproduces bit for bit:
 *   dev[n][b]  = k_{j,n}[b] - kbar_j[b]
 *   h[a*d + b] = tsum over the B rows n of (v_{j,n}[a] * dev[n][b])
 *   M_j        = sqrt(tsum over the d*d entries a*d + b of h^2)   (IEEE sqrt)
 *   bias_j     = ln_repro(M_j + eps)
 * with tsum as in pisa_select and ln_repro the fixed-operation logarithm:
 * x = 2^e m, m folded into [sqrt(1/2), sqrt(2)) (the fp32 constant 0x1.6a09e6p+0),
 * s = (m - 1)/(m + 1), t = Horner in s^2 on the fp32 constants 1/9, 1/7, 1/5, 1/3
 * and 1, ln x = e * fl(ln 2) + (t * s) * 2, every operation one IEEE fp32
 * round-to-nearest step in that order.  eps in [1e-30, 1e30]
 * (pisa_attention_ex uses PISA_ROUTE_EPS).  Output: bias [BH, nblk] fp32. */
pisa_status pisa_route_bias(const void* k, const void* v, const float* kbar, int batch, int heads, int L,
                            int d, pisa_dtype dtype, int B, float eps, float* bias, void* stream);

/* Centroids only: kbar [BH, nblk, d] fp32 of k ([BH, L, d], `dtype`), in the
 * canonical fp32 order of pisa_select (pairwise tree over the B rows, times
 * 1/B).  This is the part of the prepare phase the token-form path needs. */
pisa_status pisa_centroids(const void* k, int batch, int heads, int L, int d, pisa_dtype dtype, int B,
                           float* kbar, void* stream);

/* The fused attention kernel alone, given a selection mask from pisa_select
 * (phases 1-2 of the PISA paper's section 3.4 plus the normalisation).
 *   path PISA_PATH_STATS needs `st` (pisa_stats output with st->order >= order);
 *   path PISA_PATH_STATS_TC needs `st` with kbar, vsum, hstat and kaug (bf16,
 *   st->order >= 1) and order 1;
 *   path PISA_PATH_RECOMPUTE_TC ignores `st` (may be NULL); AUTO picks as
 *   pisa_attention does (the K it needs is taken from the mask's shape: AUTO
 *   here never picks PISA_PATH_STATS_TC, pass it explicitly).
 * mask: [BH, nblk, ceil(nblk/32)] uint32 as written by pisa_select. */
pisa_status pisa_fused_attention(const void* q, const void* k, const void* v, int batch, int heads, int L,
                                 int d, pisa_dtype dtype, int B, int order, int gate_w, pisa_path path,
                                 const uint32_t* mask, const pisa_stats_t* st, void* out, void* stream);

/* Device workspace pisa_attention needs (bytes) for the AUTO path. */
size_t pisa_workspace_bytes(int batch, int heads, int L, int d, int B, int K, int order,
                            pisa_dtype dtype);

/* Workspace for an explicit path; 0 if the path cannot run this shape. */
size_t pisa_workspace_bytes_ex(int batch, int heads, int L, int d, int B, int K, int order,
                               pisa_dtype dtype, pisa_path path);

/* Full forward pass: statistics, selection and the fused attention, enqueued
 * on `stream`.  q, k, v: [BH, L, d] of `dtype`; q pre-scaled by 1/sqrt(d).
 * out: [BH, L, d] of `dtype` (bf16 output is rounded to nearest even from fp32).
 * workspace: caller device memory of ws_bytes >= pisa_workspace_bytes(...),
 * 256-byte aligned; its contents on return are the statistics and the
 * selection of this call.  Gate on for order 2. */
pisa_status pisa_attention(const void* q, const void* k, const void* v, int batch, int heads,
                           int L, int d, pisa_dtype dtype, int B, int K, int order, void* out,
                           void* workspace, size_t ws_bytes, void* stream);

/* Bits of the gate_w argument of pisa_attention_ex and pisa_fused_attention. */
#define PISA_FLAG_GATE_W 1   /* zero w when it exceeds ln B (pisa_attention sets it) */
#define PISA_FLAG_POOLED_W 2 /* order 2: PWT's cheap form of w ("Sparse Linear Attention"
                              * blog, PWT section): w_ij = 1/2 sum_c mean_{t in tile i}(q_tc^2)
                              * var_c(keys of block j), one value per (query tile, block),
                              * instead of the exact per-query 1/2 q^T C_j q.  Required
                              * for order 2 on the hybrid path; pisa_attention_ex only. */
#define PISA_FLAG_COV_ROUTE 4 /* covariance-aware selection: pisa_route_bias with
                               * PISA_ROUTE_EPS, then pisa_select_biased (pisa_attention_ex) */
#define PISA_ROUTE_EPS 1e-6f

/* As pisa_attention with the PWT options as flags (gate_w: PISA_FLAG_GATE_W,
 * PISA_FLAG_POOLED_W, PISA_FLAG_COV_ROUTE; 0 = exact w, never zeroed, centroid
 * routing) and an explicit path.  The workspace of an order-2 call also holds
 * the pooled-w arrays; every workspace holds the routing bias. */
pisa_status pisa_attention_ex(const void* q, const void* k, const void* v, int batch, int heads,
                              int L, int d, pisa_dtype dtype, int B, int K, int order, int gate_w,
                              pisa_path path, void* out, void* workspace, size_t ws_bytes,
                              void* stream);

/* As pisa_attention_ex, plus the log of each row's denominator:
 *   lse [BH, L] fp32 (device, 4-byte aligned): lse_t = ln D_t with D_t the
 *   shared denominator of the PISA paper's section 3.2 "Formulation" (exact
 *   keys e^{q.k} plus B e^{l_tj} per unselected block), i.e. m_t + ln sum e^{. - m_t}
 *   for the kernel's running max m_t.  pisa_attention_backward_lse takes it, so
 *   that the backward needs no pass of its own over the keys for m_t and D_t.
 * Errors as pisa_attention_ex; INVALID_ARG for a null or misaligned lse;
 * UNSUPPORTED on the hybrid path. */
pisa_status pisa_attention_lse(const void* q, const void* k, const void* v, int batch, int heads, int L, int d,
                               pisa_dtype dtype, int B, int K, int order, int gate_w, pisa_path path, void* out,
                               float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Allocation-free pisa_attention (the paper has no counterpart: this is an
 * interface for callers that may not allocate device memory, such as a plugin
 * whose host application owns the whole device memory pool, or a loop where
 * cudaMalloc/cudaFree, which can synchronise the device, are not allowed).
 * Same arguments and result as pisa_attention (AUTO path, gate on), minus the
 * workspace: the scratch comes from one array of pisa_noalloc_scratch_bytes()
 * (32 MiB) compiled into the library, which every GPU that loads the library
 * holds until the process exits.  The caller still passes q, k, v and out.
 *   - No cudaMalloc, cudaFree or other allocating call is made.
 *   - The first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make that
 *     first call before any stream capture.
 *   - When the 32 MiB is committed: with CUDA's lazy module loading (the
 *     default since CUDA 12.2) the library's module, and the array with it,
 *     is loaded on a device at the library's first kernel launch or symbol
 *     lookup there, which can be this entry point's first call.  A host that
 *     hands its whole memory pool out later should make one call (or any other
 *     call of this library) on each device first, or set CUDA_MODULE_LOADING=EAGER.
 *   - The cached address belongs to the device's primary context: a
 *     cudaDeviceReset (or another teardown of that context) after the first
 *     call is not supported; the same holds for the device status word that
 *     every entry point caches.
 *   - A call whose workspace (pisa_workspace_bytes) exceeds the scratch size is
 *     rejected with PISA_ERR_INVALID_ARG before any work is enqueued.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents.  Every kernel overwrites the parts it reads, so nothing has to
 *     start at zero, but calls that overlap on the GPU (different streams, no
 *     ordering between them) race on the scratch and give wrong results. */
pisa_status pisa_attention_noalloc(const void* q, const void* k, const void* v, int batch, int heads, int L,
                                   int d, pisa_dtype dtype, int B, int K, int order, void* out, void* stream);

/* Size in bytes of the scratch array pisa_attention_noalloc uses. */
size_t pisa_noalloc_scratch_bytes(void);

/* Inputs and output in HOST memory (pinned, for the copies to overlap):
 * pisa_attention_ex over chunks of chunk_heads (batch, head) units, alternating
 * between stream0 and stream1; each chunk is copied in, computed and copied
 * back on its stream, so the copies of one chunk overlap the attention of the
 * other.  device_buf (256-byte aligned, pisa_attention_host_bytes(...) bytes,
 * caller-owned) holds two chunks of q, k, v, out and their workspaces.
 * Asynchronous: the result is in out_host once both streams have completed.
 * The operation is the same as pisa_attention_ex's (heads are independent). */
pisa_status pisa_attention_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                                int batch, int heads, int L, int d, pisa_dtype dtype, int B, int K, int order,
                                int gate_w, pisa_path path, int chunk_heads, void* device_buf,
                                size_t device_bytes, void* stream0, void* stream1);

/* Bytes of device_buf pisa_attention_host needs (0 for invalid arguments). */
size_t pisa_attention_host_bytes(int batch, int heads, int L, int d, pisa_dtype dtype, int B, int K, int order,
                                 pisa_path path, int chunk_heads);

/* Backward pass: gradients dq, dk, dv of sum_t dO_t . o_t, where o is the
 * output of pisa_attention_ex on the same q, k, v with the same B, K, order
 * and flags on the per-block (non-hybrid) paths.  The pages define only the forward
 * (PISA paper section 3.2 "Formulation"; "Sparse Linear Attention" blog,
 * sections "Sparse Linear Attention" and the PWT section); this differentiates
 * that forward with the block selection held fixed (the routing is detached,
 * as the PWT blog trains it) and, for order 2, the gate decision held fixed.
 * Per query row t, with x_n = q_t.k_n, G_n = dO_t.v_n, delta = dO_t.o_t and
 * m, D the forward's shared max and denominator:
 *   selected key n:        dS_n = P_n (G_n - delta),  P_n = e^{x_n - m}/D
 *   key n of unselected j: u_n = x_n - q_t.kbar_j,  a = e^{l_tj - m}/D,
 *                          P_n = a (1 + [order>=1] u_n),
 *                          dS_n = a (dl_n (sum_n G_n (1 + [order>=1] u_n) - B delta)
 *                                    + [order>=1] (G_n - mean_n G_n)),
 *                          dl_n = 1/B (+ u_n/B for order 2 with the gate open)
 *   dq_t = sum_n dS_tn k_n,  dk_n = sum_t dS_tn q_t,  dv_n = sum_t P_tn dO_t.
 * Arguments:
 *   q, k, v, o, dO : [BH, L, d] of `dtype`, device, 16-byte aligned; o is the
 *                    forward output (only delta = dO.o is taken from it).
 *   flags          : PISA_FLAG_GATE_W and PISA_FLAG_COV_ROUTE as in
 *                    pisa_attention_ex (the same selection is recomputed
 *                    here); PISA_FLAG_POOLED_W returns PISA_ERR_UNSUPPORTED.
 *   dq, dk, dv     : [BH, L, d] fp32 outputs, device, 8-byte aligned, fully
 *                    overwritten (no accumulation into existing contents).
 *   workspace      : ws_bytes >= pisa_backward_workspace_bytes(...) of device
 *                    memory, 256-byte aligned; on return it holds the centroids,
 *                    the selection mask and the per-row m, 1/D and delta.
 * Shapes as for pisa_attention plus batch * heads <= 65535.  bf16 inputs with
 * d and B in {64, 128} and L % 128 == 0 run on tcgen05 tensor cores: a dq
 * kernel (query-major) and a dk/dv kernel (key-major), fp32 accumulation in
 * TMEM, P and dS rounded to bf16 as the operands of the dq, dk and dv
 * products; other bf16 shapes use warp-level MMAs with the same roundings;
 * fp32 inputs run in fp32 throughout.
 * PISA_FLAG_POOLED_W (order 2; the "Sparse Linear Attention" blog, PWT section,
 * the diagonal + pooled variant): w_ij = 1/2 sum_c q2_ic var_jc of the forward,
 * recomputed here, with its gate decisions held fixed; its gradient reaches q
 * through the tile means of q^2 and k through the blocks' channel variances.
 * It runs on the tensor-core shapes and takes the forward's lse
 * (pisa_attention_backward_lse); the order-2 workspace holds its arrays.
 * Errors (before anything is enqueued): INVALID_ARG for a null or misaligned
 * pointer, unknown flag bits, K out of range, the pooled w at an order other
 * than 2, or a small workspace; UNSUPPORTED for batch * heads > 65535, the
 * pooled w off the tensor-core shapes or without lse, and the shapes
 * pisa_attention does not support. */
pisa_status pisa_attention_backward(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                    int batch, int heads, int L, int d, pisa_dtype dtype, int B, int K, int order,
                                    int flags, float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes,
                                    void* stream);

/* As pisa_attention_backward, given the forward's log-denominators lse [BH, L] fp32
 * (pisa_attention_lse on the same inputs and options; device, 4-byte aligned):
 * the backward then takes m and D from lse (P_n = e^{x_n - lse_t},
 * a = e^{l_tj - lse_t}) instead of recomputing them.  Errors as
 * pisa_attention_backward; INVALID_ARG for a null or misaligned lse. */
pisa_status pisa_attention_backward_lse(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                        const float* lse, int batch, int heads, int L, int d, pisa_dtype dtype, int B,
                                        int K, int order, int flags, float* dq, float* dk, float* dv,
                                        void* workspace, size_t ws_bytes, void* stream);

/* Workspace pisa_attention_backward needs (bytes); 0 for invalid arguments. */
size_t pisa_backward_workspace_bytes(int batch, int heads, int L, int d, int B, int K, int order,
                                     pisa_dtype dtype);

/* The path AUTO resolves to for these arguments (or -1 if none can run). */
int pisa_resolve_path(int batch, int heads, int L, int d, int B, int K, int order,
                      pisa_dtype dtype);

/* Message for the last non-OK status returned on this host thread. */
const char* pisa_last_error(void);

/* Synchronise `stream`, then read and clear the device status word of the
 * current device.  Returns PISA_ERR_DEVICE_TIMEOUT if a bounded device-side
 * wait of an earlier kernel gave up (that kernel's output is then invalid),
 * PISA_ERR_CUDA on a CUDA error, PISA_OK otherwise. */
pisa_status pisa_poll_device_status(void* stream);

/* Failure-path self-test of the bounded device waits (no counterpart on the
 * pages).  Enqueues one CTA whose single thread waits, bounded by limit_cycles
 * SM clock cycles (1 .. 2e9), on a fresh mbarrier that nothing completes, with
 * the same bounded wait the tensor-core kernels use.  The wait gives up, sets
 * the timeout bit of the device status word and the kernel exits; the next
 * pisa_poll_device_status returns PISA_ERR_DEVICE_TIMEOUT and clears the word.
 * The context stays usable.  Errors: INVALID_ARG for a limit out of range. */
pisa_status pisa_selftest_wait_timeout(long long limit_cycles, void* stream);

/* Self-test of the base-2 exponentials of the attention kernels' softmax (no
 * counterpart on the pages): y[i] = 2^x[i] for i < n, evaluated with
 * which = 0: the FMA-pipe polynomial (x = n + f, n = round(x), a cubic in
 *            f in [-1/2, 1/2] fitted for relative error <= 7.5e-5, n added to
 *            the exponent; exactly 0 for x <= -125; valid up to x = 64), or
 * which = 1: the special-function unit's ex2.approx.ftz.
 * x, y: fp32 device arrays of n elements, 4-byte aligned.  Errors:
 * INVALID_ARG for n < 0, which not 0 or 1, a null or misaligned pointer. */
pisa_status pisa_selftest_ex2(const float* x, float* y, long long n, int which, void* stream);

/* Library version string. */
const char* pisa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PISA_H_ */
