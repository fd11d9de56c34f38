"""CPU oracle for piecewise sparse attention (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and it imports nothing
from the product.

Thin ctypes wrapper over ``pisa_oracle.cpp`` (fp64 math, canonical fp32
selection).  All arrays are numpy, C-contiguous, layout [BH, L, d].
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = ctypes.c_void_p
        li = ctypes.c_long
        L.oracle_block_stats.argtypes = [f32p, f32p, li, li, li, li, f64p, f64p, f64p, f64p, ctypes.c_int]
        L.oracle_select.argtypes = [f32p, f32p, li, li, li, li, li, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        L.oracle_route_bias.argtypes = [f32p, f32p, li, li, li, li, ctypes.c_float, ctypes.c_void_p, ctypes.c_int]
        L.oracle_ln_f32.argtypes = [f32p, li, ctypes.c_void_p]
        L.oracle_pisa_attention.argtypes = [f32p, f32p, f32p, li, li, li, li, li, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_void_p, li, f64p, f64p, ctypes.c_int]
        L.oracle_pisa_hybrid.argtypes = [f32p, f32p, f32p, li, li, li, li, li, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_void_p, li, f64p, f64p, ctypes.c_int]
        L.oracle_pisa_attention_ex.argtypes = [f32p, f32p, f32p, li, li, li, li, li, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                               ctypes.c_void_p, li, f64p, f64p, ctypes.c_int]
        L.oracle_pisa_bruteforce.argtypes = [f32p, f32p, f32p, li, li, li, li, li, ctypes.c_int,
                                             ctypes.c_int, f64p, ctypes.c_int]
        L.oracle_centroids_f32.argtypes = [f32p, li, li, li, li, ctypes.c_void_p, ctypes.c_int]
        L.oracle_dense_attention.argtypes = [f32p, f32p, f32p, li, li, li, f64p, ctypes.c_int]
        L.oracle_pisa_backward.argtypes = [f32p, f32p, f32p, f32p, ctypes.c_void_p, li, li, li, li, li,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, f64p, f64p,
                                           f64p, ctypes.c_int]
        L.oracle_pisa_backward_dq_rows.argtypes = [f32p, f32p, f32p, f32p, ctypes.c_void_p, li, li, li, li, li,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_void_p, li,
                                                   f64p, ctypes.c_int]
        for fn in ("oracle_pisa_backward", "oracle_pisa_backward_dq_rows", "oracle_route_bias", "oracle_ln_f32", "oracle_pisa_attention_ex", "oracle_pisa_hybrid", "oracle_centroids_f32", "oracle_block_stats", "oracle_select", "oracle_pisa_attention",
                   "oracle_pisa_bruteforce", "oracle_dense_attention"):
            getattr(L, fn).restype = ctypes.c_int
        _lib = L
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected the shape/arguments")


def block_stats(k, v, B, order=2, nthreads=None):
    """fp64 (kbar [BH,nblk,d], vsum [BH,nblk,d], H [BH,nblk,d,d] or None, C or None).

    H[bh, j, a, b] = sum_n v[n, a] * (k[n, b] - kbar[b]);  C = (1/B) sum_n dev dev^T.
    """
    k, v = _f32(k), _f32(v)
    BH, L, d = k.shape
    nblk = L // B
    kbar = np.zeros((BH, nblk, d))
    vsum = np.zeros((BH, nblk, d))
    H = np.zeros((BH, nblk, d, d)) if order >= 1 else None
    C = np.zeros((BH, nblk, d, d)) if order == 2 else None
    rc = lib().oracle_block_stats(k, v, BH, L, d, B, _ptr(kbar), _ptr(vsum), _ptr(H), _ptr(C),
                                  nthreads or default_threads())
    _check(rc, "block_stats")
    return kbar, vsum, H, C


def centroids_f32(k, B, nthreads=None):
    """Canonical fp32 key centroids [BH, nblk, d] (tree sum times 1/B), as used by the selection."""
    k = _f32(k)
    BH, L, d = k.shape
    out = np.zeros((BH, L // B, d), np.float32)
    rc = lib().oracle_centroids_f32(k, BH, L, d, B, _ptr(out), nthreads or default_threads())
    _check(rc, "centroids_f32")
    return out


def ln_f32(x):
    """The reproducible fp32 natural logarithm the routing bias uses (element-wise)."""
    x = _f32(x)
    out = np.zeros_like(x)
    _check(lib().oracle_ln_f32(x.ravel(), x.size, _ptr(out)), "ln_f32")
    return out


def route_bias(k, v, B, eps=1e-6, nthreads=None):
    """Covariance-aware routing bias ln(||H_j||_F + eps), canonical fp32, [BH, nblk]."""
    k, v = _f32(k), _f32(v)
    BH, L, d = k.shape
    out = np.zeros((BH, L // B), np.float32)
    rc = lib().oracle_route_bias(k, v, BH, L, d, B, float(eps), _ptr(out), nthreads or default_threads())
    _check(rc, "route_bias")
    return out


def select(q, k, B, K, nthreads=None, want_scores=False, bias=None):
    """Canonical fp32 selection: (idx [BH,nblk,K] int32 ascending, mask [BH,nblk,words] uint32,
    scores [BH,nblk,nblk] float32 or None).  With ``bias`` ([BH, nblk] fp32) every score
    s_ij becomes s_ij + bias_j (one fp32 add) before the top-K."""
    q, k = _f32(q), _f32(k)
    if bias is not None:
        bias = _f32(bias)
    BH, L, d = q.shape
    nblk = L // B
    words = (nblk + 31) // 32
    idx = np.zeros((BH, nblk, K), np.int32)
    mask = np.zeros((BH, nblk, words), np.uint32)
    scores = np.zeros((BH, nblk, nblk), np.float32) if want_scores else None
    rc = lib().oracle_select(q, k, BH, L, d, B, K, _ptr(idx), _ptr(mask), _ptr(scores), _ptr(bias),
                             nthreads or default_threads())
    _check(rc, "select")
    return idx, mask, scores


def _attention(fn, q, k, v, B, K, order, gate, tiles, nthreads, want_lse):
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, L, d = q.shape
    nblk = L // B
    full = tiles is None
    if full:
        tl = np.array([(bh, i) for bh in range(BH) for i in range(nblk)], dtype=np.int64)
    else:
        tl = np.ascontiguousarray(np.asarray(tiles, dtype=np.int64).reshape(-1, 2))
    out = np.zeros((tl.shape[0], B, d))
    lse = np.zeros((tl.shape[0], B)) if want_lse else None
    rc = fn(q, k, v, BH, L, d, B, K, int(order), int(bool(gate)), _ptr(tl), tl.shape[0], _ptr(out), _ptr(lse),
            nthreads or default_threads())
    _check(rc, "attention")
    if full:
        out = out.reshape(BH, L, d)
        lse = lse.reshape(BH, L) if want_lse else None
    return (out, lse) if want_lse else out


def pisa_hybrid(q, k, v, B, K, order=1, gate=True, tiles=None, nthreads=None, want_lse=False):
    """PISA hybrid output: as pisa_attention but the first-order term uses the
    global H-bar = (B/L) sum_j H_j of each (batch, head) for every unselected
    block (same return convention as pisa_attention)."""
    return _attention(lib().oracle_pisa_hybrid, q, k, v, B, K, order, gate, tiles, nthreads, want_lse)


def pisa_attention_ex(q, k, v, B, K, order=1, gate=True, hybrid=False, w_pooled=False, route_eps=None, tiles=None,
                      nthreads=None, want_lse=False):
    """General form: ``hybrid`` uses the global H-bar (PISA hybrid), ``w_pooled``
    PWT's diagonal + pooled second-order correction (order 2), ``route_eps`` (a
    positive float) the covariance-aware selection with bias ln(||H_j||_F + eps)."""
    fn = lib().oracle_pisa_attention_ex
    reps = float(route_eps) if route_eps else 0.0

    def call(q_, k_, v_, BH, L, d, B_, K_, o_, g_, tl, n, out, lse, nt):
        return fn(q_, k_, v_, BH, L, d, B_, K_, o_, g_, int(bool(hybrid)), int(bool(w_pooled)), reps, tl, n, out,
                  lse, nt)

    return _attention(call, q, k, v, B, K, order, gate, tiles, nthreads, want_lse)


def pisa_attention(q, k, v, B, K, order=1, gate=True, tiles=None, nthreads=None, want_lse=False):
    """Statistics-form output.  With tiles=None returns [BH, L, d] fp64; otherwise
    ``tiles`` is a sequence of (bh, i) query tiles and the result is [ntiles, B, d].
    With want_lse the log-denominator log(D_t) is returned too (same leading shape)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, L, d = q.shape
    nblk = L // B
    full = tiles is None
    if full:
        tl = np.array([(bh, i) for bh in range(BH) for i in range(nblk)], dtype=np.int64)
    else:
        tl = np.ascontiguousarray(np.asarray(tiles, dtype=np.int64).reshape(-1, 2))
    out = np.zeros((tl.shape[0], B, d))
    lse = np.zeros((tl.shape[0], B)) if want_lse else None
    rc = lib().oracle_pisa_attention(q, k, v, BH, L, d, B, K, int(order), int(bool(gate)),
                                     _ptr(tl), tl.shape[0], _ptr(out), _ptr(lse),
                                     nthreads or default_threads())
    _check(rc, "pisa_attention")
    if full:
        out = out.reshape(BH, L, d)
        lse = lse.reshape(BH, L) if want_lse else None
    return (out, lse) if want_lse else out


def pisa_bruteforce(q, k, v, B, K, order=1, gate=True, nthreads=None):
    """Token-wise first-order form without block statistics, [BH, L, d] fp64."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, L, d = q.shape
    out = np.zeros((BH, L, d))
    rc = lib().oracle_pisa_bruteforce(q, k, v, BH, L, d, B, K, int(order), int(bool(gate)),
                                      _ptr(out), nthreads or default_threads())
    _check(rc, "pisa_bruteforce")
    return out


def pisa_backward(q, k, v, dO, B, K, order=1, gate=True, route_eps=None, nthreads=None, o=None, w_pooled=False):
    """(dq, dk, dv) [BH, L, d] fp64: gradients of sum_t dO_t . o_t for pisa_attention's
    output o, with the block selection held fixed (``route_eps``: the covariance-aware
    selection, as in pisa_attention_ex).  ``o``: None (delta_t = dO_t . o_t from the
    recomputed fp64 output) or the forward output the caller holds ([BH, L, d], taken as
    fp32), as a backward operator of (q, k, v, o, dO) receives it.  ``w_pooled`` (order 2):
    the output of pisa_attention_ex(..., w_pooled=True), PWT's diagonal + pooled w, with its
    gate decisions held fixed."""
    q, k, v, dO = _f32(q), _f32(k), _f32(v), _f32(dO)
    BH, L, d = q.shape
    og = None if o is None else _f32(o)
    if og is not None and og.shape != q.shape:
        raise ValueError("o must have q's shape")
    dq, dk, dv = (np.zeros((BH, L, d)) for _ in range(3))
    reps = float(route_eps) if route_eps else 0.0
    rc = lib().oracle_pisa_backward(q, k, v, dO, _ptr(og), BH, L, d, B, K, int(order), int(bool(gate)),
                                    int(bool(w_pooled)), reps, _ptr(dq), _ptr(dk), _ptr(dv),
                                    nthreads or default_threads())
    _check(rc, "pisa_backward")
    return dq, dk, dv


def pisa_backward_dq_rows(q, k, v, dO, B, K, rows, order=1, gate=True, route_eps=None, nthreads=None, o=None):
    """dq of the query rows ``rows`` (a sequence of (bh, t)), [nrows, d] fp64: the same
    rows of pisa_backward's dq, computed one row at a time (for sampled checks at sizes
    where the whole backward is too slow on the CPU); ``o`` as in pisa_backward."""
    q, k, v, dO = _f32(q), _f32(k), _f32(v), _f32(dO)
    BH, L, d = q.shape
    og = None if o is None else _f32(o)
    if og is not None and og.shape != q.shape:
        raise ValueError("o must have q's shape")
    rl = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    out = np.zeros((rl.shape[0], d))
    reps = float(route_eps) if route_eps else 0.0
    rc = lib().oracle_pisa_backward_dq_rows(q, k, v, dO, _ptr(og), BH, L, d, B, K, int(order), int(bool(gate)), reps,
                                            _ptr(rl), rl.shape[0], _ptr(out), nthreads or default_threads())
    _check(rc, "pisa_backward_dq_rows")
    return out


def dense_attention(q, k, v, nthreads=None):
    """softmax(q k^T) v in fp64, [BH, L, d]."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, L, d = q.shape
    out = np.zeros((BH, L, d))
    rc = lib().oracle_dense_attention(q, k, v, BH, L, d, _ptr(out), nthreads or default_threads())
    _check(rc, "dense_attention")
    return out


def rel_l2(a, b) -> float:
    """||a - b||_F / ||b||_F."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def parity_metrics(got, ref, row_floor=0.0) -> dict:
    """Comparison figures of a result ``got`` against the oracle's ``ref`` (same shape; the
    last axis is one output row):
      rel_l2   ||got - ref||_F / ||ref||_F over everything compared;
      row_max  max over rows t of ||got_t - ref_t|| / max(||ref_t||, row_floor rms_row), rms_row
               the rms of the rows' reference norms (row_floor 0: the plain relative error; a
               gradient row can cancel to nearly nothing, and its relative error then means
               little, so gradients are compared with row_floor 1).  Rows whose reference norm
               is below 1e-6 of rms_row are skipped when row_floor is 0;
      row_worst the index of that row in the flattened row list (-1 if none);
      elem_max max over elements of |got - ref| / (rms(ref) + |ref|), rms over everything
               compared, i.e. the smallest e with |got - ref| <= e rms(ref) + e |ref| everywhere;
      rows     the number of rows compared."""
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    if g.shape != r.shape:
        raise ValueError(f"shape mismatch {g.shape} vs {r.shape}")
    d = g.shape[-1] if g.ndim else 1
    g2, r2 = g.reshape(-1, d), r.reshape(-1, d)
    diff = g2 - r2
    rn = np.linalg.norm(r2, axis=1)
    dn = np.linalg.norm(diff, axis=1)
    rms_row = float(np.sqrt(np.mean(rn * rn))) if rn.size else 0.0
    live = rn > 1e-6 * max(rms_row, 1e-300) if row_floor <= 0 else np.ones(rn.shape, bool)
    den = np.maximum(rn, row_floor * rms_row)
    row_err = dn[live] / den[live] if live.any() else np.zeros(0)
    rms = float(np.sqrt(np.mean(r2 * r2))) if r2.size else 0.0
    ratio = np.abs(diff) / (rms + np.abs(r2) + 1e-300)
    worst = int(np.argmax(row_err)) if row_err.size else -1
    return {
        "rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(r2), 1e-300)),
        "row_max": float(row_err.max()) if row_err.size else 0.0,
        "row_worst": int(np.flatnonzero(live)[worst]) if worst >= 0 else -1,
        "elem_max": float(ratio.max()) if ratio.size else 0.0,
        "rows": int(r2.shape[0]),
    }


LN = math.log
