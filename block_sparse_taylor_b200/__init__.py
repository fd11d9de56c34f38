"""Python binding of the B200 piecewise sparse attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libpisa_b200.so`` (C ABI in ``include/pisa.h``).  PyTorch is used
for device memory and streams.  There is no fallback: if the compiled library
is missing, importing a function raises ``PisaLibraryMissing``; build it with
``python -m block_sparse_taylor_b200.build``.

The functions carry the names of the C entry points:

* ``pisa_stats(k, v, B, order)``: block statistics (centroids, value sums,
  H_j, C_j), the prepare phase of the PISA paper (section 3.4, Figure 3).
* ``pisa_select(q, stats, K)``: per query tile, the top-K key blocks by the
  tile-mean query's centroid score, reproducible bit for bit.
* ``pisa_attention(q, k, v, B, K, order)``: the full forward pass of piecewise
  sparse attention (PISA paper section 3.2; "Sparse Linear Attention" blog,
  PWT section for order 2).
* ``pisa_attention_backward(q, k, v, o, dO, B, K, order)``: dq, dk, dv of that
  forward with the block selection held fixed; ``pisa_attention_autograd`` wraps
  both as a torch.autograd.Function.

Tensors are [batch*heads, L, d] (or [batch, heads, L, d]) contiguous CUDA
tensors of dtype float32 or bfloat16; q must already be multiplied by
1/sqrt(d).
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libpisa_b200.so")

PISA_OK, PISA_ERR_INVALID_ARG, PISA_ERR_UNSUPPORTED, PISA_ERR_CUDA, PISA_ERR_DEVICE_TIMEOUT = range(5)
PISA_F32, PISA_BF16 = 0, 1
PATHS = {"auto": 0, "stats": 1, "recompute_tc": 2, "hybrid_tc": 3, "stats_tc": 4}
FLAG_GATE_W, FLAG_POOLED_W, FLAG_COV_ROUTE = 1, 2, 4
ROUTE_EPS = 1e-6
PATH_NAMES = {v: k for k, v in PATHS.items()}


class PisaLibraryMissing(ImportError):
    pass


class PisaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"pisa status {status}: {msg}")
        self.status = status


class _StatsT(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("heads", ctypes.c_int), ("L", ctypes.c_int), ("d", ctypes.c_int),
                ("B", ctypes.c_int), ("nblk", ctypes.c_int), ("order", ctypes.c_int), ("dtype", ctypes.c_int),
                ("kbar", ctypes.c_void_p), ("vsum", ctypes.c_void_p), ("hstat", ctypes.c_void_p),
                ("cov", ctypes.c_void_p), ("kaug", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded CUDA library (raises PisaLibraryMissing if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise PisaLibraryMissing(f"{LIB_PATH} not found: run `python -m block_sparse_taylor_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i, sz, vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
        L.pisa_version.restype = ctypes.c_char_p
        L.pisa_last_error.restype = ctypes.c_char_p
        L.pisa_stats_bytes.argtypes = [i, i, i, i, i, i, i]
        L.pisa_stats_bytes.restype = sz
        L.pisa_stats_bind.argtypes = [ctypes.POINTER(_StatsT), vp, sz, i, i, i, i, i, i, i]
        L.pisa_stats.argtypes = [vp, vp, ctypes.POINTER(_StatsT), vp]
        L.pisa_select.argtypes = [vp, ctypes.POINTER(_StatsT), i, vp, vp, vp]
        L.pisa_select_biased.argtypes = [vp, ctypes.POINTER(_StatsT), i, vp, vp, vp, vp]
        L.pisa_select_scores.argtypes = [vp, ctypes.POINTER(_StatsT), vp, vp, vp]
        L.pisa_route_bias.argtypes = [vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, vp, vp]
        L.pisa_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
        L.pisa_workspace_bytes.restype = sz
        L.pisa_workspace_bytes_ex.argtypes = [i, i, i, i, i, i, i, i, i]
        L.pisa_workspace_bytes_ex.restype = sz
        L.pisa_attention.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, i, vp, vp, sz, vp]
        L.pisa_attention_ex.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, i, i, i, vp, vp, sz, vp]
        L.pisa_resolve_path.argtypes = [i, i, i, i, i, i, i, i]
        L.pisa_poll_device_status.argtypes = [vp]
        L.pisa_centroids.argtypes = [vp, i, i, i, i, i, i, vp, vp]
        L.pisa_fused_attention.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, i, i, vp, ctypes.POINTER(_StatsT),
                                           vp, vp]
        L.pisa_attention_noalloc.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, i, vp, vp]
        L.pisa_attention_host.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, i, vp, sz, vp, vp]
        L.pisa_attention_host.restype = ctypes.c_int
        L.pisa_attention_host_bytes.argtypes = [i, i, i, i, i, i, i, i, i, i]
        L.pisa_attention_host_bytes.restype = sz
        L.pisa_noalloc_scratch_bytes.restype = sz
        L.pisa_attention_backward.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, vp, vp, vp, vp, sz, vp]
        L.pisa_attention_backward.restype = ctypes.c_int
        L.pisa_attention_backward_lse.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, vp, vp, vp, vp,
                                                  sz, vp]
        L.pisa_attention_backward_lse.restype = ctypes.c_int
        L.pisa_attention_lse.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, i, i, i, vp, vp, vp, sz, vp]
        L.pisa_attention_lse.restype = ctypes.c_int
        L.pisa_backward_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
        L.pisa_backward_workspace_bytes.restype = sz
        L.pisa_selftest_wait_timeout.argtypes = [ctypes.c_longlong, vp]
        L.pisa_selftest_wait_timeout.restype = ctypes.c_int
        L.pisa_selftest_ex2.argtypes = [vp, vp, ctypes.c_longlong, i, vp]
        L.pisa_selftest_ex2.restype = ctypes.c_int
        for fn in ("pisa_attention_noalloc", "pisa_centroids", "pisa_fused_attention", "pisa_stats_bind", "pisa_stats", "pisa_select", "pisa_attention", "pisa_attention_ex",
                   "pisa_poll_device_status", "pisa_resolve_path"):
            getattr(L, fn).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status != PISA_OK:
        raise PisaError(status, lib().pisa_last_error().decode())


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return PISA_BF16
    if t == torch.float32:
        return PISA_F32
    raise TypeError(f"unsupported dtype {t}")


def _shape(x: torch.Tensor):
    if x.dim() == 4:
        return x.shape[0], x.shape[1], x.shape[2], x.shape[3]
    if x.dim() == 3:
        return 1, x.shape[0], x.shape[1], x.shape[2]
    raise ValueError("expected [batch, heads, L, d] or [batch*heads, L, d]")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")


def version() -> str:
    return lib().pisa_version().decode()


class Stats(NamedTuple):
    kbar: torch.Tensor            # [BH, nblk, d] fp32
    vsum: torch.Tensor            # [BH, nblk, d] fp32
    hstat: Optional[torch.Tensor]  # [BH, nblk, d, d] (rows = value channel)
    cov: Optional[torch.Tensor]    # [BH, nblk, d, d]
    raw: _StatsT
    buf: torch.Tensor
    kaug: Optional[torch.Tensor] = None  # [BH, nblk, 8, d] bf16: high and low parts of kbar, zero rows


def pisa_stats_bytes(batch, heads, L, d, B, order, dtype: torch.dtype) -> int:
    return int(lib().pisa_stats_bytes(batch, heads, L, d, B, order, _dtype_code(dtype)))


def pisa_stats(k: torch.Tensor, v: torch.Tensor, B: int, order: int = 2, buf: Optional[torch.Tensor] = None,
               stream=None) -> Stats:
    """Block statistics of k, v (prepare phase).  Returns views into ``buf``."""
    _need_cuda(k, v)
    batch, heads, L, d = _shape(k)
    code = _dtype_code(k.dtype)
    nbytes = pisa_stats_bytes(batch, heads, L, d, B, order, k.dtype)
    if nbytes == 0:
        raise PisaError(PISA_ERR_INVALID_ARG, "invalid dimensions for pisa_stats")
    if buf is None:
        buf = torch.empty(nbytes, dtype=torch.uint8, device=k.device)
    st = _StatsT()
    _check(lib().pisa_stats_bind(ctypes.byref(st), buf.data_ptr(), buf.numel(), batch, heads, L, d, B, order, code))
    _check(lib().pisa_stats(k.data_ptr(), v.data_ptr(), ctypes.byref(st), _stream(stream)))
    return _stats_views(st, buf, k.dtype)


def _stats_views(st: _StatsT, buf: torch.Tensor, dtype: torch.dtype) -> Stats:
    BH = st.batch * st.heads
    base = buf.data_ptr()

    def view(ptr, shape, dt):
        if not ptr:
            return None
        n = 1
        for s in shape:
            n *= s
        off = ptr - base
        es = torch.empty((), dtype=dt).element_size()
        return buf[off:off + n * es].view(dt).view(*shape)

    kbar = view(st.kbar, (BH, st.nblk, st.d), torch.float32)
    vsum = view(st.vsum, (BH, st.nblk, st.d), torch.float32)
    hstat = view(st.hstat, (BH, st.nblk, st.d, st.d), dtype)
    cov = view(st.cov, (BH, st.nblk, st.d, st.d), dtype)
    kaug = view(st.kaug, (BH, st.nblk, 8, st.d), torch.bfloat16)
    return Stats(kbar, vsum, hstat, cov, st, buf, kaug)


def pisa_centroids(k: torch.Tensor, B: int, kbar: Optional[torch.Tensor] = None, stream=None) -> Stats:
    """Canonical fp32 centroids only (what the selection needs); returns a Stats
    whose other arrays are None."""
    _need_cuda(k)
    batch, heads, L, d = _shape(k)
    if kbar is None:
        kbar = torch.empty((batch * heads, L // B, d), dtype=torch.float32, device=k.device)
    _check(lib().pisa_centroids(k.data_ptr(), batch, heads, L, d, _dtype_code(k.dtype), B, kbar.data_ptr(),
                                _stream(stream)))
    st = _StatsT(batch, heads, L, d, B, L // B, 0, _dtype_code(k.dtype), kbar.data_ptr(), None, None, None, None)
    return Stats(kbar, None, None, None, st, kbar)


def pisa_fused_attention(q, k, v, B: int, mask: torch.Tensor, order: int = 1, gate: bool = True,
                         path: str = "auto", stats: Optional[Stats] = None, out: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """The fused attention kernel alone, given the selection mask of pisa_select."""
    _need_cuda(q, k, v, mask)
    batch, heads, L, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    st = ctypes.byref(stats.raw) if stats is not None else None
    _check(lib().pisa_fused_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), batch, heads, L, d,
                                      _dtype_code(q.dtype), B, order, int(bool(gate)), PATHS[path],
                                      mask.data_ptr(), st, out.data_ptr(), _stream(stream)))
    return out


def pisa_route_bias(k: torch.Tensor, v: torch.Tensor, kbar: torch.Tensor, B: int, eps: float = ROUTE_EPS,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Covariance-aware routing bias ln(||H_j||_F + eps), [BH, nblk] fp32 (kbar: the
    canonical centroids of pisa_centroids / pisa_stats)."""
    _need_cuda(k, v, kbar)
    batch, heads, L, d = _shape(k)
    if out is None:
        out = torch.empty((batch * heads, L // B), dtype=torch.float32, device=k.device)
    _check(lib().pisa_route_bias(k.data_ptr(), v.data_ptr(), kbar.data_ptr(), batch, heads, L, d,
                                 _dtype_code(k.dtype), B, float(eps), out.data_ptr(), _stream(stream)))
    return out


def pisa_select(q: torch.Tensor, stats: Stats, K: int, stream=None, bias: Optional[torch.Tensor] = None):
    """(idx [BH, nblk, K] int32 ascending, mask [BH, nblk, ceil(nblk/32)] int32 bit words).
    With ``bias`` ([BH, nblk] fp32, e.g. pisa_route_bias) the covariance-aware selection."""
    _need_cuda(q)
    st = stats.raw
    BH = st.batch * st.heads
    words = (st.nblk + 31) // 32
    idx = torch.empty((BH, st.nblk, max(K, 0)), dtype=torch.int32, device=q.device)
    mask = torch.empty((BH, st.nblk, words), dtype=torch.int32, device=q.device)
    if bias is None:
        _check(lib().pisa_select(q.data_ptr(), ctypes.byref(st), K, idx.data_ptr() if K > 0 else None,
                                 mask.data_ptr(), _stream(stream)))
    else:
        _need_cuda(bias)
        _check(lib().pisa_select_biased(q.data_ptr(), ctypes.byref(st), K, bias.data_ptr(),
                                        idx.data_ptr() if K > 0 else None, mask.data_ptr(), _stream(stream)))
    return idx, mask


def _flags(gate: bool, w_mode: str, route: str) -> int:
    if w_mode not in ("exact", "pooled"):
        raise ValueError(f"w_mode must be 'exact' or 'pooled' (got {w_mode!r})")
    if route not in ("centroid", "cov"):
        raise ValueError(f"route must be 'centroid' or 'cov' (got {route!r})")
    return ((FLAG_GATE_W if gate else 0) | (FLAG_POOLED_W if w_mode == "pooled" else 0)
            | (FLAG_COV_ROUTE if route == "cov" else 0))


def pisa_select_scores(q: torch.Tensor, stats: Stats, bias: Optional[torch.Tensor] = None, stream=None):
    """The selection's fp32 score table [BH, nblk, nblk] (row = query tile), as the top-K sees it."""
    _need_cuda(q)
    st = stats.raw
    scores = torch.empty((st.batch * st.heads, st.nblk, st.nblk), dtype=torch.float32, device=q.device)
    _check(lib().pisa_select_scores(q.data_ptr(), ctypes.byref(st), None if bias is None else bias.data_ptr(),
                                    scores.data_ptr(), _stream(stream)))
    return scores


def pisa_workspace_bytes(batch, heads, L, d, B, K, order, dtype: torch.dtype, path: str = "auto") -> int:
    return int(lib().pisa_workspace_bytes_ex(batch, heads, L, d, B, K, order, _dtype_code(dtype), PATHS[path]))


def pisa_resolve_path(batch, heads, L, d, B, K, order, dtype: torch.dtype) -> str:
    p = lib().pisa_resolve_path(batch, heads, L, d, B, K, order, _dtype_code(dtype))
    if p < 0:
        raise PisaError(PISA_ERR_INVALID_ARG, "no path for these arguments")
    return PATH_NAMES[p]


def pisa_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, B: int, K: int, order: int = 1,
                   gate: bool = True, path: str = "auto", out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None, w_mode: str = "exact",
                   route: str = "centroid") -> torch.Tensor:
    """Piecewise sparse attention forward; returns ``out`` (same shape and dtype as q).
    ``w_mode`` ("exact" or "pooled") picks the order-2 correction: the exact
    1/2 q^T C_j q, or PWT's diagonal + pooled [query tile x block] estimate.
    ``route`` ("centroid" or "cov") picks the selection score: the centroid score,
    or the covariance-aware score plus ln(||H_j||_F + ROUTE_EPS)."""
    _need_cuda(q, k, v)
    if not (q.shape == k.shape == v.shape and q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share shape and dtype")
    batch, heads, L, d = _shape(q)
    code = _dtype_code(q.dtype)
    if out is None:
        out = torch.empty_like(q)
    _need_cuda(out)
    nbytes = pisa_workspace_bytes(batch, heads, L, d, B, K, order, q.dtype, path)
    if nbytes == 0:
        raise PisaError(PISA_ERR_INVALID_ARG if path == "auto" else PISA_ERR_UNSUPPORTED,
                        f"no workspace size for these arguments (path={path})")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _check(lib().pisa_attention_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), batch, heads, L, d, code, B, K,
                                   order, _flags(gate, w_mode, route),
                                   PATHS[path], out.data_ptr(), workspace.data_ptr(),
                                   workspace.numel(), _stream(stream)))
    return out


def pisa_attention_lse(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, B: int, K: int, order: int = 1,
                       gate: bool = True, path: str = "auto", out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None,
                       w_mode: str = "exact", route: str = "centroid"):
    """pisa_attention plus each row's log-denominator: returns (out, lse) with lse [batch*heads, L]
    fp32, lse_t = ln D_t (what pisa_attention_backward takes to skip its own row statistics)."""
    _need_cuda(q, k, v)
    if not (q.shape == k.shape == v.shape and q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share shape and dtype")
    batch, heads, L, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((batch * heads, L), dtype=torch.float32, device=q.device)
    _need_cuda(out, lse)
    nbytes = pisa_workspace_bytes(batch, heads, L, d, B, K, order, q.dtype, path)
    if nbytes == 0:
        raise PisaError(PISA_ERR_INVALID_ARG if path == "auto" else PISA_ERR_UNSUPPORTED,
                        f"no workspace size for these arguments (path={path})")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _check(lib().pisa_attention_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), batch, heads, L, d,
                                    _dtype_code(q.dtype), B, K, order, _flags(gate, w_mode, route), PATHS[path],
                                    out.data_ptr(), lse.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                    _stream(stream)))
    return out, lse


def pisa_backward_workspace_bytes(batch, heads, L, d, B, K, order, dtype: torch.dtype) -> int:
    return int(lib().pisa_backward_workspace_bytes(batch, heads, L, d, B, K, order, _dtype_code(dtype)))


def pisa_attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, dO: torch.Tensor,
                            B: int, K: int, order: int = 1, gate: bool = True, route: str = "centroid",
                            grads: Optional[tuple] = None, workspace: Optional[torch.Tensor] = None, stream=None,
                            lse: Optional[torch.Tensor] = None, w_mode: str = "exact"):
    """(dq, dk, dv) fp32, the gradients of sum(dO * o) for o = pisa_attention(q, k, v, B, K, order,
    gate=gate, route=route, w_mode=w_mode) on the per-block paths, the selection held fixed.
    ``o`` is that forward's output; ``lse`` optionally its log-denominators (pisa_attention_lse),
    which spares the backward its own pass for the row statistics (the pooled w, order 2,
    requires it); ``grads`` optional preallocated fp32 (dq, dk, dv)."""
    _need_cuda(q, k, v, o, dO)
    if not (q.shape == k.shape == v.shape == o.shape == dO.shape
            and q.dtype == k.dtype == v.dtype == o.dtype == dO.dtype):
        raise ValueError("q, k, v, o, dO must share shape and dtype")
    batch, heads, L, d = _shape(q)
    code = _dtype_code(q.dtype)
    if grads is None:
        grads = tuple(torch.empty(q.shape, dtype=torch.float32, device=q.device) for _ in range(3))
    for g in grads:
        _need_cuda(g)
        if g.dtype != torch.float32 or g.shape != q.shape:
            raise ValueError("grads must be fp32 tensors of q's shape")
    nbytes = pisa_backward_workspace_bytes(batch, heads, L, d, B, K, order, q.dtype)
    if nbytes == 0:
        raise PisaError(PISA_ERR_INVALID_ARG, "no backward workspace size for these arguments")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    dq, dk, dv = grads
    if lse is None:
        _check(lib().pisa_attention_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dO.data_ptr(),
                                             batch, heads, L, d, code, B, K, order, _flags(gate, w_mode, route),
                                             dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                                             workspace.numel(), _stream(stream)))
    else:
        _need_cuda(lse)
        if lse.dtype != torch.float32 or lse.numel() != batch * heads * L:
            raise ValueError("lse must be fp32 with batch*heads*L elements")
        _check(lib().pisa_attention_backward_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                                 dO.data_ptr(), lse.data_ptr(), batch, heads, L, d, code, B, K, order,
                                                 _flags(gate, w_mode, route), dq.data_ptr(), dk.data_ptr(),
                                                 dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                                 _stream(stream)))
    return dq, dk, dv


class PisaAttentionFunction(torch.autograd.Function):
    """pisa_attention as a torch.autograd.Function: the forward is pisa_attention, the backward
    pisa_attention_backward (selection held fixed); gradients are returned in the inputs' dtype."""

    @staticmethod
    def forward(ctx, q, k, v, B, K, order, gate, path, route, w_mode):
        out, lse = pisa_attention_lse(q, k, v, B, K, order, gate=gate, path=path, route=route, w_mode=w_mode)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.cfg = (B, K, order, gate, route, w_mode)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        B, K, order, gate, route, w_mode = ctx.cfg
        dq, dk, dv = pisa_attention_backward(q, k, v, out, dout.contiguous(), B, K, order, gate=gate, route=route,
                                             lse=lse, w_mode=w_mode)
        return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), None, None, None, None, None, None, None


def pisa_attention_autograd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, B: int, K: int, order: int = 1,
                            gate: bool = True, path: str = "auto", route: str = "centroid",
                            w_mode: str = "exact") -> torch.Tensor:
    """pisa_attention with gradients for training (the per-block paths: "auto", "recompute_tc",
    "stats", "stats_tc"; exact w, or PWT's pooled w at order 2 on the tensor-core shapes).  The
    backward holds the block selection (and the gate decisions) fixed."""
    if path == "hybrid_tc":
        raise PisaError(PISA_ERR_UNSUPPORTED, "no backward for the hybrid path")
    return PisaAttentionFunction.apply(q, k, v, B, K, order, gate, path, route, w_mode)


def pisa_attention_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, B: int, K: int, order: int = 1,
                           out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """pisa_attention without a workspace argument, for callers that may not
    allocate device memory: the library's built-in scratch array is used (see
    include/pisa.h).  ``out`` must be given by such callers (it is created
    here only for convenience when omitted)."""
    _need_cuda(q, k, v)
    batch, heads, L, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().pisa_attention_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), batch, heads, L, d,
                                        _dtype_code(q.dtype), B, K, order, out.data_ptr(), _stream(stream)))
    return out


class HostPlan:
    """Device staging and streams for pisa_attention_host (allocated once)."""

    def __init__(self, q: torch.Tensor, B: int, K: int, order: int = 1, path: str = "auto", chunk_heads: int = 4,
                 device: Optional[torch.device] = None):
        batch, heads, L, d = _shape(q)
        self.args = (batch, heads, L, d, _dtype_code(q.dtype), B, K, order)
        self.path, self.chunk = path, chunk_heads
        nbytes = int(lib().pisa_attention_host_bytes(batch, heads, L, d, _dtype_code(q.dtype), B, K, order,
                                                     PATHS[path], chunk_heads))
        if nbytes == 0:
            raise PisaError(PISA_ERR_INVALID_ARG, "no host plan for these arguments")
        dev = device or torch.device("cuda", torch.cuda.current_device())
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.streams = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))


def pisa_attention_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, plan: HostPlan,
                        gate: bool = True, w_mode: str = "exact", route: str = "centroid"):
    """pisa_attention on pinned host tensors (q, k, v, out on the CPU); the work
    is queued on the plan's two streams, which the caller synchronises."""
    for t in (q, k, v, out):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("pisa_attention_host takes contiguous host tensors")
    batch, heads, L, d, code, B, K, order = plan.args
    flags = _flags(gate, w_mode, route)
    _check(lib().pisa_attention_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), batch, heads, L, d,
                                     code, B, K, order, flags, PATHS[plan.path], plan.chunk, plan.buf.data_ptr(),
                                     plan.buf.numel(), plan.streams[0].cuda_stream, plan.streams[1].cuda_stream))


def pisa_selftest_wait_timeout(limit_cycles: int = 2_000_000, stream=None):
    """Enqueue the failure-path self-test: a bounded device wait that runs out (see
    include/pisa.h).  The next pisa_poll_device_status raises PisaError with status
    PISA_ERR_DEVICE_TIMEOUT."""
    _check(lib().pisa_selftest_wait_timeout(int(limit_cycles), _stream(stream)))


def pisa_selftest_ex2(x: torch.Tensor, which: str = "fma", out: Optional[torch.Tensor] = None, stream=None):
    """y = 2^x element-wise with one of the kernels' exponentials: "fma" (the FMA-pipe
    polynomial) or "sfu" (ex2.approx); x a contiguous fp32 CUDA tensor."""
    _need_cuda(x)
    if x.dtype != torch.float32:
        raise TypeError("pisa_selftest_ex2 takes float32")
    if out is None:
        out = torch.empty_like(x)
    _check(lib().pisa_selftest_ex2(x.data_ptr(), out.data_ptr(), x.numel(), {"fma": 0, "sfu": 1}[which],
                                   _stream(stream)))
    return out


def pisa_poll_device_status(stream=None):
    """Synchronise and raise PisaError if a device-side bounded wait gave up."""
    _check(lib().pisa_poll_device_status(_stream(stream)))
