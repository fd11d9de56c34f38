"""Host-side checks of the C ABI: the library loads, exports every entry point
declared in include/pisa.h, and rejects bad arguments before touching a GPU.

These run without a GPU: validation happens before any CUDA call, so the
pointers passed here are never dereferenced.
"""
import ctypes
import os
import re

import pytest

import block_sparse_taylor_b200 as pisa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b(pisa_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pisa_stats", "pisa_select", "pisa_attention", "pisa_workspace_bytes", "pisa_last_error",
                     "pisa_poll_device_status", "pisa_stats_bind", "pisa_stats_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(pisa.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_version_string():
    assert pisa.version().startswith("pisa-b200")


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first


def call_ex(L=1024, d=64, B=64, K=4, order=1, dtype=pisa.PISA_BF16, path=0, ws_bytes=1 << 30, batch=1, heads=1,
            q=FAKE, ws=FAKE):
    return pisa.lib().pisa_attention_ex(q, FAKE, FAKE, batch, heads, L, d, dtype, B, K, order, 1, path, FAKE, ws,
                                        ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(L=1000), pisa.PISA_ERR_INVALID_ARG),          # L % B
    (dict(K=17), pisa.PISA_ERR_INVALID_ARG),            # K > nblk
    (dict(K=-1), pisa.PISA_ERR_INVALID_ARG),
    (dict(order=3), pisa.PISA_ERR_INVALID_ARG),
    (dict(dtype=7), pisa.PISA_ERR_INVALID_ARG),
    (dict(batch=0), pisa.PISA_ERR_INVALID_ARG),
    (dict(d=96), pisa.PISA_ERR_UNSUPPORTED),
    (dict(B=32, L=1024), pisa.PISA_ERR_UNSUPPORTED),
    (dict(q=None), pisa.PISA_ERR_INVALID_ARG),
    (dict(ws=None), pisa.PISA_ERR_INVALID_ARG),
    (dict(ws_bytes=16), pisa.PISA_ERR_INVALID_ARG),
    (dict(ws=ctypes.c_void_p(0x1008)), pisa.PISA_ERR_INVALID_ARG),  # misaligned workspace
    (dict(path=9), pisa.PISA_ERR_INVALID_ARG),
    (dict(path=2, dtype=pisa.PISA_F32), pisa.PISA_ERR_UNSUPPORTED),  # tensor cores need bf16
    (dict(path=3, order=2), pisa.PISA_ERR_UNSUPPORTED),              # the hybrid has orders 0 and 1
    (dict(L=1024 * 8192, B=64), pisa.PISA_ERR_UNSUPPORTED),          # nblk > 4096
])
def test_bad_arguments_are_rejected_before_launch(kw, status):
    assert call_ex(**kw) == status
    assert len(pisa.lib().pisa_last_error()) > 0


def test_workspace_sizes_and_paths():
    bf, f32 = pisa.PISA_BF16, pisa.PISA_F32
    lib = pisa.lib()
    # fp32 can only take the statistics path
    assert lib.pisa_resolve_path(1, 1, 1024, 64, 64, 4, 1, f32) == pisa.PATHS["stats"]
    assert lib.pisa_resolve_path(1, 40, 32768, 128, 64, 77, 1, bf) == pisa.PATHS["recompute_tc"]
    assert lib.pisa_resolve_path(1, 1, 1000, 64, 64, 4, 1, bf) == -1
    ws_stats = lib.pisa_workspace_bytes_ex(1, 12, 8192, 64, 64, 16, 2, bf, 1)
    ws_tc = lib.pisa_workspace_bytes_ex(1, 12, 8192, 64, 64, 16, 2, bf, 2)
    # the statistics path holds H_j and C_j (2 x 12 x 128 x 64 x 64 bf16), the recompute path does not
    assert ws_stats - ws_tc >= 2 * 12 * 128 * 64 * 64 * 2
    assert lib.pisa_workspace_bytes_ex(1, 1, 1024, 64, 64, 4, 1, f32, 2) == 0
    assert lib.pisa_workspace_bytes(1, 1, 1024, 64, 64, 4, 1, f32) == lib.pisa_workspace_bytes_ex(
        1, 1, 1024, 64, 64, 4, 1, f32, 1)


def test_auto_takes_the_association_with_fewer_flops():
    # d = B = 128 (Hunyuan shape) and d = B = 64 (clustered shape), order 1: the statistics form on
    # the tensor cores executes fewer FLOPs than the token form's 4 L d per row; d = 2B (Wan and
    # FLUX shapes) and any order-2 call with the exact w keep the token form
    bf = pisa.PISA_BF16
    lib = pisa.lib()
    st = pisa.PATHS["stats_tc"]
    assert lib.pisa_resolve_path(1, 24, 118784, 128, 128, 93, 1, bf) == st
    assert lib.pisa_resolve_path(1, 12, 8192, 64, 64, 16, 1, bf) == st
    assert lib.pisa_resolve_path(1, 12, 8192, 64, 64, 16, 2, bf) == pisa.PATHS["recompute_tc"]
    assert lib.pisa_resolve_path(1, 40, 32768, 128, 64, 77, 1, bf) == pisa.PATHS["recompute_tc"]
    assert lib.pisa_resolve_path(1, 24, 4608, 128, 64, 36, 1, bf) == pisa.PATHS["recompute_tc"]
    # with every block selected there is no statistics term, and the token form costs the same: token
    assert lib.pisa_resolve_path(1, 12, 8192, 64, 64, 128, 1, bf) == pisa.PATHS["recompute_tc"]
    # the statistics-form workspace holds H_j and the centroid split (no C_j), order 0 has no such path
    ws = lib.pisa_workspace_bytes_ex(1, 12, 8192, 64, 64, 16, 1, bf, st)
    ws_tok = lib.pisa_workspace_bytes_ex(1, 12, 8192, 64, 64, 16, 1, bf, 2)
    assert ws - ws_tok >= 12 * 128 * (64 * 64 + 8 * 64) * 2 + 12 * 128 * 64 * 4
    assert lib.pisa_workspace_bytes_ex(1, 12, 8192, 64, 64, 16, 0, bf, st) == 0
    assert lib.pisa_workspace_bytes_ex(1, 12, 8192, 64, 64, 16, 1, pisa.PISA_F32, st) == 0
    assert lib.pisa_workspace_bytes_ex(1, 12, 8192, 64, 64, 16, 2, bf, st) > ws  # pooled w arrays


def test_statistics_form_path_rejects_what_it_cannot_run():
    # order 2 needs the pooled w; order 0 has no statistics term; fp32 has no tensor-core path
    assert call_ex(path=4, order=2) == pisa.PISA_ERR_UNSUPPORTED
    assert call_ex(path=4, order=0) == pisa.PISA_ERR_UNSUPPORTED
    assert call_ex(path=4, dtype=pisa.PISA_F32) == pisa.PISA_ERR_UNSUPPORTED


def test_stats_bind_layout():
    st = pisa._StatsT()
    lib = pisa.lib()
    n = lib.pisa_stats_bytes(2, 3, 1024, 64, 64, 2, pisa.PISA_BF16)
    assert n >= 2 * 6 * 16 * 64 * 4 + 2 * 6 * 16 * 64 * 64 * 2
    base = 0x10000
    assert lib.pisa_stats_bind(ctypes.byref(st), ctypes.c_void_p(base), n, 2, 3, 1024, 64, 64, 2, pisa.PISA_BF16) == 0
    assert st.nblk == 16 and st.kbar == base and st.cov is not None and st.hstat is not None
    assert (st.vsum - base) % 256 == 0 and (st.hstat - base) % 256 == 0 and (st.cov - base) % 256 == 0
    assert lib.pisa_stats_bind(ctypes.byref(st), ctypes.c_void_p(base), n - 1, 2, 3, 1024, 64, 64, 2,
                               pisa.PISA_BF16) == pisa.PISA_ERR_INVALID_ARG
    assert (st.kaug - base) % 256 == 0 and st.kaug >= st.cov + 6 * 16 * 64 * 64 * 2
    assert lib.pisa_stats_bind(ctypes.byref(st), ctypes.c_void_p(base), n, 2, 3, 1024, 64, 64, 1, pisa.PISA_BF16) == 0
    assert st.cov is None and st.kaug is not None
    # the centroid split exists only for bf16 statistics of order >= 1
    n0 = lib.pisa_stats_bytes(2, 3, 1024, 64, 64, 0, pisa.PISA_BF16)
    assert lib.pisa_stats_bind(ctypes.byref(st), ctypes.c_void_p(base), n0, 2, 3, 1024, 64, 64, 0, pisa.PISA_BF16) == 0
    assert st.kaug is None
    nf = lib.pisa_stats_bytes(2, 3, 1024, 64, 64, 1, pisa.PISA_F32)
    assert lib.pisa_stats_bind(ctypes.byref(st), ctypes.c_void_p(base), nf, 2, 3, 1024, 64, 64, 1, pisa.PISA_F32) == 0
    assert st.kaug is None


def test_routing_and_score_entry_points_reject_bad_arguments():
    lib = pisa.lib()
    bf = pisa.PISA_BF16
    # eps outside [1e-30, 1e30], null pointers, a bad shape: rejected before any CUDA call
    for eps in (0.0, -1.0, 1e31, float("nan")):
        assert lib.pisa_route_bias(FAKE, FAKE, FAKE, 1, 1, 1024, 64, bf, 64, eps, FAKE, None) == \
            pisa.PISA_ERR_INVALID_ARG
    assert lib.pisa_route_bias(None, FAKE, FAKE, 1, 1, 1024, 64, bf, 64, 1e-6, FAKE, None) == pisa.PISA_ERR_INVALID_ARG
    assert lib.pisa_route_bias(FAKE, FAKE, FAKE, 1, 1, 1000, 64, bf, 64, 1e-6, FAKE, None) == pisa.PISA_ERR_INVALID_ARG
    assert lib.pisa_route_bias(FAKE, FAKE, FAKE, 1, 1, 1024, 96, bf, 64, 1e-6, FAKE, None) == pisa.PISA_ERR_UNSUPPORTED
    st = pisa._StatsT(1, 1, 1024, 64, 64, 16, 0, bf, FAKE.value, None, None, None, None)
    assert lib.pisa_select_scores(FAKE, ctypes.byref(st), None, None, None) == pisa.PISA_ERR_INVALID_ARG
    assert lib.pisa_select_scores(None, ctypes.byref(st), None, FAKE, None) == pisa.PISA_ERR_INVALID_ARG
    assert lib.pisa_select_biased(FAKE, ctypes.byref(st), 17, FAKE, FAKE, FAKE, None) == pisa.PISA_ERR_INVALID_ARG
    assert lib.pisa_select_biased(FAKE, ctypes.byref(st), 4, FAKE, None, None, None) == pisa.PISA_ERR_INVALID_ARG
    assert lib.pisa_select_scores(FAKE, None, None, FAKE, None) == pisa.PISA_ERR_INVALID_ARG


def test_binding_flags():
    assert pisa._flags(True, "exact", "centroid") == pisa.FLAG_GATE_W
    assert pisa._flags(False, "pooled", "cov") == pisa.FLAG_POOLED_W | pisa.FLAG_COV_ROUTE
    for bad in (("exact", "nope"), ("nope", "centroid")):
        with pytest.raises(ValueError):
            pisa._flags(True, *bad)


def test_workspace_holds_the_routing_bias():
    # the routing bias is part of every workspace: enabling the flag never needs more
    for path in ("recompute_tc", "hybrid_tc", "stats"):
        n = pisa.pisa_workspace_bytes(1, 2, 2048, 128, 64, 8, 1, pisa.torch.bfloat16, path)
        assert n > 2 * (2048 // 64) * 4


def call_bwd(L=1024, d=64, B=64, K=4, order=1, dtype=pisa.PISA_BF16, flags=1, ws_bytes=1 << 30, batch=1, heads=1,
             q=FAKE, o=FAKE, dq=FAKE, ws=FAKE):
    return pisa.lib().pisa_attention_backward(q, FAKE, FAKE, o, FAKE, batch, heads, L, d, dtype, B, K, order, flags,
                                              dq, FAKE, FAKE, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(L=1000), pisa.PISA_ERR_INVALID_ARG),                  # L % B
    (dict(K=17), pisa.PISA_ERR_INVALID_ARG),                    # K > nblk
    (dict(order=3), pisa.PISA_ERR_INVALID_ARG),
    (dict(d=96), pisa.PISA_ERR_UNSUPPORTED),
    (dict(flags=8), pisa.PISA_ERR_INVALID_ARG),                 # unknown flag bit
    (dict(flags=pisa.FLAG_POOLED_W), pisa.PISA_ERR_INVALID_ARG),  # the pooled w is an order-2 option
    (dict(batch=2, heads=40000), pisa.PISA_ERR_UNSUPPORTED),    # grid y limit
    (dict(q=None), pisa.PISA_ERR_INVALID_ARG),
    (dict(o=None), pisa.PISA_ERR_INVALID_ARG),
    (dict(dq=None), pisa.PISA_ERR_INVALID_ARG),
    (dict(q=ctypes.c_void_p(0x1008)), pisa.PISA_ERR_INVALID_ARG),   # inputs need 16-byte alignment
    (dict(dq=ctypes.c_void_p(0x1004)), pisa.PISA_ERR_INVALID_ARG),  # gradients need 8-byte alignment
    (dict(ws=None), pisa.PISA_ERR_INVALID_ARG),
    (dict(ws=ctypes.c_void_p(0x1010)), pisa.PISA_ERR_INVALID_ARG),  # workspace needs 256-byte alignment
    (dict(ws_bytes=64), pisa.PISA_ERR_INVALID_ARG),
])
def test_backward_rejects_bad_arguments_before_launch(kw, status):
    assert call_bwd(**kw) == status
    assert pisa.lib().pisa_last_error()


def test_backward_workspace_size():
    f = pisa.lib().pisa_backward_workspace_bytes
    # centroids + bias + mask + four per-row arrays (m, 1/D, delta, lse), each rounded up to 256 bytes
    BH, L, d, B = 2, 1024, 64, 64
    nblk = L // B
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    want = up(4 * BH * nblk * d) + up(4 * BH * nblk) + up(4 * BH * nblk * 1) + 4 * up(4 * BH * L)
    assert f(1, BH, L, d, B, 4, 1, pisa.PISA_BF16) == want
    assert f(1, 1, 1000, 64, 64, 4, 1, pisa.PISA_BF16) == 0
    assert f(1, 1, 1024, 64, 64, 17, 1, pisa.PISA_BF16) == 0
    # order 2 adds the pooled w's arrays: var, q2 [BH, nblk, d]; w, W [BH, nblk, nblk];
    # the per-32-row partial sums [BH, L / 32, nblk]
    pooled = 2 * up(4 * BH * nblk * d) + 2 * up(4 * BH * nblk * nblk) + up(4 * BH * (L // 32) * nblk)
    assert f(1, BH, L, d, B, 4, 2, pisa.PISA_BF16) == want + pooled


def test_pooled_w_backward_rejects_what_it_cannot_run():
    # host checks before anything touches the device: the pooled w is an order-2 option, runs
    # on the tensor-core shapes and takes the forward's lse
    L = pisa.lib()
    ws = ctypes.c_void_p(0x100000)
    args = lambda order, dt, flags: (None, None, None, None, None, 1, 1, 1024, 64, dt, 64, 4, order,  # noqa: E731
                                     flags, None, None, None, ws, 1 << 30, None)
    pooled = pisa.FLAG_POOLED_W | pisa.FLAG_GATE_W
    assert L.pisa_attention_backward(*args(1, pisa.PISA_BF16, pooled)) == pisa.PISA_ERR_INVALID_ARG
    assert L.pisa_attention_backward(*args(2, pisa.PISA_F32, pooled)) == pisa.PISA_ERR_UNSUPPORTED
    assert L.pisa_attention_backward(*args(2, pisa.PISA_BF16, pooled)) == pisa.PISA_ERR_UNSUPPORTED
    assert "lse" in L.pisa_last_error().decode()


MIS = ctypes.c_void_p(0x1008)  # 8-byte but not 16-byte aligned; never dereferenced


def test_forward_entry_points_reject_misaligned_device_arrays():
    L = pisa.lib()
    args = (1, 1, 1024, 64, pisa.PISA_BF16, 64, 4, 1)
    assert L.pisa_attention_ex(MIS, FAKE, FAKE, *args, 1, 0, FAKE, FAKE, 1 << 30, None) == pisa.PISA_ERR_INVALID_ARG
    assert L.pisa_attention_ex(FAKE, FAKE, FAKE, *args, 1, 0, MIS, FAKE, 1 << 30, None) == pisa.PISA_ERR_INVALID_ARG
    assert "16-byte" in L.pisa_last_error().decode()
    assert L.pisa_centroids(MIS, 1, 1, 1024, 64, pisa.PISA_BF16, 64, FAKE, None) == pisa.PISA_ERR_INVALID_ARG
    assert L.pisa_centroids(FAKE, 1, 1, 1024, 64, pisa.PISA_BF16, 64, MIS, None) == pisa.PISA_ERR_INVALID_ARG
    assert L.pisa_route_bias(FAKE, MIS, FAKE, 1, 1, 1024, 64, pisa.PISA_BF16, 64, ctypes.c_float(1e-6), FAKE,
                             None) == pisa.PISA_ERR_INVALID_ARG
    assert L.pisa_fused_attention(FAKE, FAKE, MIS, 1, 1, 1024, 64, pisa.PISA_BF16, 64, 1, 1, 2, FAKE, None, FAKE,
                                  None) == pisa.PISA_ERR_INVALID_ARG
    st = pisa._StatsT(1, 1, 1024, 64, 64, 16, 0, pisa.PISA_BF16, MIS.value, None, None, None)
    assert L.pisa_select(FAKE, ctypes.byref(st), 4, FAKE, FAKE, None) == pisa.PISA_ERR_INVALID_ARG
    assert L.pisa_select_biased(FAKE, ctypes.byref(st), 4, FAKE, FAKE, FAKE, None) == pisa.PISA_ERR_INVALID_ARG
    assert L.pisa_select_scores(FAKE, ctypes.byref(st), None, FAKE, None) == pisa.PISA_ERR_INVALID_ARG
    st.kbar = FAKE.value
    assert L.pisa_select(MIS, ctypes.byref(st), 4, FAKE, FAKE, None) == pisa.PISA_ERR_INVALID_ARG


def test_selftest_wait_timeout_rejects_limits_out_of_range():
    f = pisa.lib().pisa_selftest_wait_timeout
    for bad in (0, -5, 2_000_000_001):
        assert f(bad, None) == pisa.PISA_ERR_INVALID_ARG
        assert b"limit_cycles" in pisa.lib().pisa_last_error()
