"""GPU parity: every kernel of the library against the CPU oracle.

* statistics: centroids bit-exact (canonical fp32), sums and d x d statistics
  within the storage precision;
* selection: index lists and masks bit-exact, on small shapes, planted ties and
  every full-size workload;
* attention: relative L2 error (||gpu - oracle||_F / ||oracle||_F) at most 1e-4
  on the fp32 path and 2e-2 on the bf16 path, and the same bound on every row
  and (relative to the output's rms) on every element (tests/parity.py), on
  small shapes end to end and on sampled query tiles (first, last and seeded
  random ones) of the full-size workloads, through every formulation.
"""
import functools
import math

import numpy as np
import pytest
import torch

import block_sparse_taylor_b200 as pisa
import oracle
import parity
import pisa_synth

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev(x, dt):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(TDT[dt])


@functools.lru_cache(maxsize=3)
def workload(name):
    w = pisa_synth.workloads()[name]
    return w, pisa_synth.generate(w)


def sample_tiles(BH, nblk, per_head, seed, heads=None):
    rng = np.random.default_rng(seed)
    hs = range(BH) if heads is None else heads
    out = []
    for bh in hs:
        pick = {0, nblk - 1}
        while len(pick) < min(per_head, nblk):
            pick.add(int(rng.integers(0, nblk)))
        out += [(bh, i) for i in sorted(pick)]
    return out


def rows_of(o, tiles, B):
    return np.stack([o[bh, i * B:(i + 1) * B] for bh, i in tiles])


def rel_l2(a, b):
    return oracle.rel_l2(a, b)


def rows_clear_of_the_gate(q, k, B, K):
    """[BH, L] bool: rows none of whose unselected blocks has w_tj = 1/2 q_t^T C_j q_t (fp64,
    from the oracle's statistics) within 2^-8 of 1/2 |q_t|^T |C_j| |q_t| of ln B, twice the
    worst-case error of C_j's entries rounded to bf16 (2^-9 each).  The gate is a step at
    w = ln B, and the CUDA-core statistics path reads C_j in bf16: a row with a block that close
    to the threshold can take the other branch of the gate on the GPU and change by a factor of
    up to e^{ln B} on that block.  Such rows are ill-conditioned, not wrong; they are left to
    the pooled bound."""
    _, _, _, C = oracle.block_stats(k, k, B, order=2)
    _, mask, _ = oracle.select(q, k, B, K)
    BH, L, d = q.shape
    nblk = L // B
    lnb = math.log(B)
    keep = np.ones((BH, L), bool)
    bits = np.unpackbits(mask.view(np.uint8), axis=-1, bitorder="little")[:, :, :nblk].astype(bool)
    for bh in range(BH):
        q64 = q[bh].astype(np.float64)
        w = 0.5 * np.einsum("ld,jde,le->lj", q64, C[bh], q64)
        wabs = 0.5 * np.einsum("ld,jde,le->lj", np.abs(q64), np.abs(C[bh]), np.abs(q64))
        near = (np.abs(w - lnb) <= 2.0 ** -8 * wabs) & ~bits[bh][np.arange(L) // B]
        keep[bh] = ~near.any(axis=1)
    return keep


def check_gated(got, ref, q, k, B, K, what):
    """The pooled bound on every row; the row and element bounds on the rows clear of the gate
    threshold (rows_clear_of_the_gate), which must be most of them."""
    keep = rows_clear_of_the_gate(q, k, B, K)
    assert keep.mean() > 0.8, keep.mean()
    assert rel_l2(got, ref) <= TOL["bf16"]
    parity.check(got[keep], ref[keep], "bf16", what)


# ---------------------------------------------------------------------------
# statistics
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("order", [1, 2])
def test_stats_parity(dt, d, B, order):
    q, k, v = pisa_synth.random_qkv(100 + d + B, 2, 1024, d, dtype=dt)
    st = pisa.pisa_stats(dev(k, dt), dev(v, dt), B, order)
    torch.cuda.synchronize()
    kbar_ref = oracle.centroids_f32(k, B)
    assert np.array_equal(st.kbar.cpu().numpy().view(np.uint32), kbar_ref.view(np.uint32))
    _, vsum, H, C = oracle.block_stats(k, v, B, order=2)
    parity.check(st.vsum.cpu().numpy(), vsum, dt, "vsum", tol=1e-6, row_tol=1e-6, elem_tol=1e-6)
    # H_j and C_j are stored in the input dtype: bf16 rounding of every entry
    tol = 1e-5 if dt == "f32" else 8e-3
    parity.check(st.hstat.float().cpu().numpy(), H, dt, "H", tol=tol, row_tol=2 * tol, elem_tol=2 * tol)
    if order == 2:
        parity.check(st.cov.float().cpu().numpy(), C, dt, "C", tol=tol, row_tol=2 * tol, elem_tol=2 * tol)
    else:
        assert st.cov is None


@pytest.mark.parametrize("d,B,order", [(128, 64, 1), (128, 128, 2), (64, 64, 2), (64, 128, 1)])
def test_stats_parity_many_blocks_per_cta(d, B, order):
    # more blocks than SMs: every persistent CTA loops over several blocks, through the ring
    # of stages and both TMEM buffers; also the bf16 high/low split of the centroids
    q, k, v = pisa_synth.random_qkv(150 + d + B, 6, 8192, d, dtype="bf16")
    st = pisa.pisa_stats(dev(k, "bf16"), dev(v, "bf16"), B, order)
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    kbar_ref = oracle.centroids_f32(k, B)
    assert np.array_equal(st.kbar.cpu().numpy().view(np.uint32), kbar_ref.view(np.uint32))
    _, vsum, H, C = oracle.block_stats(k, v, B, order=2)
    parity.check(st.vsum.cpu().numpy(), vsum, "bf16", "vsum", tol=1e-6, row_tol=1e-6, elem_tol=1e-6)
    parity.check(st.hstat.float().cpu().numpy(), H, "bf16", "H", tol=8e-3, row_tol=1.6e-2, elem_tol=1.6e-2)
    if order == 2:
        parity.check(st.cov.float().cpu().numpy(), C, "bf16", "C", tol=8e-3, row_tol=1.6e-2, elem_tol=1.6e-2)
    ka = st.kaug.float().cpu().numpy()
    hi = pisa_synth.round_bf16(kbar_ref)
    assert np.array_equal(ka[:, :, 0], hi)
    assert np.array_equal(ka[:, :, 1], pisa_synth.round_bf16(kbar_ref - hi))
    assert not np.any(ka[:, :, 2:])


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------

def gpu_select(q, k, B, K, dt):
    st = pisa.pisa_stats(dev(k, dt), dev(k, dt), B, 0)
    idx, mask = pisa.pisa_select(dev(q, dt), st, K)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), mask.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d,B,L", [(64, 64, 2048), (128, 64, 4096), (128, 128, 4096), (64, 128, 1024),
                                   (128, 64, 2560), (64, 64, 4608), (128, 128, 1152)])
@pytest.mark.parametrize("Kfrac", [0.0, 0.1, 0.5, 1.0])
def test_select_parity(dt, d, B, L, Kfrac):
    nblk = L // B
    K = int(round(Kfrac * nblk))
    q, k, _ = pisa_synth.random_qkv(200 + d + L, 3, L, d, scale=4.0, dtype=dt)
    idx, mask = gpu_select(q, k, B, K, dt)
    ridx, rmask, _ = oracle.select(q, k, B, K)
    assert np.array_equal(mask, rmask)
    assert np.array_equal(idx, ridx)


def test_select_planted_ties():
    # Key blocks whose centroids are exact multiples of unit vectors and query
    # tiles whose means are exact, so that many scores tie exactly; the lower
    # block index must win.
    d, B, L = 64, 64, 64 * 16
    nblk = L // B
    rng = np.random.default_rng(5)
    k = np.zeros((1, L, d), np.float32)
    q = np.zeros((1, L, d), np.float32)
    for j in range(nblk):
        k[0, j * B:(j + 1) * B, j % 3] = float(1 + (j % 2))
        q[0, j * B:(j + 1) * B, rng.integers(0, 3)] = 1.0
    for K in (1, 3, 5, 8):
        idx, mask = gpu_select(q, k, B, K, "f32")
        ridx, rmask, _ = oracle.select(q, k, B, K)
        assert np.array_equal(idx, ridx) and np.array_equal(mask, rmask)


@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (128, 128)])
def test_select_near_ties_decided_by_the_canonical_scores(d, B):
    # every key block is one base block plus a perturbation of a few ulp of a single entry,
    # so the scores of a row differ by less than the approximate scores' error bound: the
    # selection must fall back to the canonical scores for most blocks and still match
    L = 2048
    nblk = L // B
    rng = np.random.default_rng(31 + d + B)
    base = rng.standard_normal((B, d)).astype(np.float32)
    k = np.tile(base, (nblk, 1))[None].copy()
    for j in range(nblk):
        c = int(rng.integers(d))
        toward = np.float32(np.inf) if j % 2 else np.float32(-np.inf)
        k[0, j * B:(j + 1) * B, c] = np.nextafter(k[0, j * B:(j + 1) * B, c], toward)
    q = rng.standard_normal((1, L, d)).astype(np.float32)
    for K in (1, nblk // 4, nblk // 2, nblk - 1):
        idx, mask = gpu_select(q, k, B, K, "f32")
        ridx, rmask, _ = oracle.select(q, k, B, K)
        assert np.array_equal(idx, ridx) and np.array_equal(mask, rmask)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d,B,L", [(64, 64, 2048), (128, 64, 4096), (128, 128, 4096), (64, 128, 1024)])
def test_select_scores_bit_exact(dt, d, B, L):
    # the canonical fp32 score table itself, not only the top-K it decides
    q, k, v = pisa_synth.random_qkv(250 + d + B + L, 2, L, d, scale=1.0, dtype=dt)
    st = pisa.pisa_centroids(dev(k, dt), B)
    sc = pisa.pisa_select_scores(dev(q, dt), st)
    torch.cuda.synchronize()
    _, _, ref = oracle.select(q, k, B, 1, want_scores=True)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("name,heads", [("c3", 4), ("c4", 2), ("c2", 12), ("c5_L16896_s90", 4)])
def test_select_scores_full_size_bit_exact(name, heads):
    w = pisa_synth.workloads()[name].with_(heads=heads)
    q, k, v = pisa_synth.generate(w)
    st = pisa.pisa_centroids(dev(k, w.dtype), w.B)
    sc = pisa.pisa_select_scores(dev(q, w.dtype), st)
    torch.cuda.synchronize()
    _, _, ref = oracle.select(q, k, w.B, 1, want_scores=True)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4", "c5_L4608_s75", "c5_L16896_s90"])
def test_select_full_size(name):
    w, (q, k, v) = workload(name)
    idx, mask = gpu_select(q, k, w.B, w.K, w.dtype)
    ridx, rmask, _ = oracle.select(q, k, w.B, w.K)
    assert np.array_equal(mask, rmask)
    assert np.array_equal(idx, ridx)


# ---------------------------------------------------------------------------
# attention, small shapes, whole output
# ---------------------------------------------------------------------------

def run_attn(q, k, v, B, K, order, dt, path="auto", gate=True):
    out = pisa.pisa_attention(dev(q, dt), dev(k, dt), dev(v, dt), B, K, order, gate=gate, path=path)
    pisa.pisa_poll_device_status()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("path", ["stats", "recompute_tc"])
@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("order", [0, 1, 2])
def test_attention_small_bf16(path, d, B, order):
    L = 1024
    q, k, v = pisa_synth.random_qkv(300 + d + B + order, 2, L, d, scale=2.0, dtype="bf16")
    K = (L // B) // 4
    got = run_attn(q, k, v, B, K, order, "bf16", path)
    ref = oracle.pisa_attention(q, k, v, B, K, order)
    m = parity.check(got, ref, "bf16")
    assert m["rel_l2"] <= 5e-3, m  # the expected bf16 rounding level; a formulation slip is far above it


@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("order", [0, 1, 2])
def test_attention_small_f32(d, B, order):
    L = 1024
    q, k, v = pisa_synth.random_qkv(400 + d + B + order, 2, L, d, scale=2.0, dtype="f32")
    K = (L // B) // 4
    got = run_attn(q, k, v, B, K, order, "f32")
    ref = oracle.pisa_attention(q, k, v, B, K, order)
    parity.check(got, ref, "f32")


def test_attention_c1_fp32():
    w, (q, k, v) = workload("c1")
    got = run_attn(q, k, v, w.B, w.K, w.order, w.dtype)
    ref = oracle.pisa_attention(q, k, v, w.B, w.K, w.order)
    parity.check(got, ref, "f32")


@pytest.mark.parametrize("path", ["stats", "recompute_tc"])
@pytest.mark.parametrize("case", ["K0", "Kall", "ragged", "batched", "sharp", "gate"])
def test_attention_edge_cases(path, case):
    d, B, L, BH, K, order, scale = 128, 64, 1024, 2, 4, 1, 2.0
    batch = 1
    if case == "K0":
        K = 0
    elif case == "Kall":
        K = L // B
    elif case == "ragged":
        L = 1152  # 4.5 CTAs of 256 rows: the last CTA has one live 128-row tile
    elif case == "batched":
        batch, BH = 2, 6
    elif case == "sharp":
        scale = 8.0  # large logits: exercises the running-max correction
    q, k, v = pisa_synth.random_qkv(500 + len(case), BH, L, d, scale=scale, dtype="bf16")
    if case == "gate":
        order = 2
        k[:, :, 7] *= 30.0  # an outlier channel: w exceeds ln B on many blocks
        k = pisa_synth.round_bf16(k)
    qt, kt, vt = (dev(x, "bf16") for x in (q, k, v))
    if batch > 1:
        qt, kt, vt = (x.view(batch, BH // batch, L, d) for x in (qt, kt, vt))
    got = pisa.pisa_attention(qt, kt, vt, B, K, order, path=path).float().cpu().numpy().reshape(BH, L, d)
    pisa.pisa_poll_device_status()
    ref = oracle.pisa_attention(q, k, v, B, K, order)
    if case == "gate":
        check_gated(got, ref, q, k, B, K, case)
    else:
        parity.check(got, ref, "bf16", case)
    if case == "Kall":
        parity.check(got, oracle.dense_attention(q, k, v), "bf16", "dense")


def test_gate_changes_the_result_when_w_is_large():
    d, B, L = 64, 64, 1024
    q, k, v = pisa_synth.random_qkv(600, 1, L, d, scale=2.0, dtype="bf16")
    k[:, :, 3] *= 30.0
    k = pisa_synth.round_bf16(k)
    for path in ("stats", "recompute_tc"):
        on = run_attn(q, k, v, B, 4, 2, "bf16", path, gate=True)
        off = run_attn(q, k, v, B, 4, 2, "bf16", path, gate=False)
        check_gated(on, oracle.pisa_attention(q, k, v, B, 4, 2, gate=True), q, k, B, 4, "gate on")
        # With the gate off, w reaches several hundred on these inputs (that is what the
        # scaled key column is for), and a row's output follows e^w of its largest block:
        # the statistics path's bf16 C_j moves w by up to 2^-9 (1/2 |q|^T |C_j| |q|), over
        # 2^-5 on every row here.  Such rows are ill-conditioned, so the gate-off arm keeps
        # the pooled bound only; the gate-on arm (w <= ln B) has all three.
        assert rel_l2(off, oracle.pisa_attention(q, k, v, B, 4, 2, gate=False)) <= TOL["bf16"]
        assert rel_l2(on, off) > 1e-2


# ---------------------------------------------------------------------------
# attention, full-size workloads, sampled tiles
# ---------------------------------------------------------------------------

FULL = [("c2", "recompute_tc", 1, 6), ("c2o2", "recompute_tc", 1, 6), ("c2", "stats", 1, 6),
        ("c2o2", "stats", 1, 6), ("c3", "recompute_tc", 2, None), ("c4", "recompute_tc", 1, 8),
        ("c5_L4608_s50", "recompute_tc", 2, None), ("c5_L4608_s75", "recompute_tc", 2, None),
        ("c5_L4608_s90", "recompute_tc", 2, None), ("c5_L4608_s95", "recompute_tc", 2, None),
        ("c5_L16896_s50", "recompute_tc", 2, 8), ("c5_L16896_s75", "recompute_tc", 2, 8),
        ("c5_L16896_s90", "recompute_tc", 2, 8), ("c5_L16896_s95", "recompute_tc", 2, 8),
        ("c2", "stats_tc", 1, 6), ("c4", "stats_tc", 1, 8), ("c3", "stats_tc", 1, 8),
        ("c5_L16896_s90", "stats_tc", 2, 8), ("c5_L4608_s50", "stats_tc", 2, None)]


@pytest.mark.parametrize("name,path,per_head,nheads", FULL)
def test_attention_full_size_sampled(name, path, per_head, nheads):
    w, (q, k, v) = workload(name)
    got = run_attn(q, k, v, w.B, w.K, w.order, w.dtype, path)
    heads = None if nheads is None else list(np.random.default_rng(7).choice(w.BH, nheads, replace=False))
    tiles = sample_tiles(w.BH, w.nblk, per_head, seed=11, heads=heads)
    ref = oracle.pisa_attention(q, k, v, w.B, w.K, w.order, tiles=tiles)
    parity.check(rows_of(got, tiles, w.B), ref, w.dtype, name)


def test_device_status_is_clean():
    q, k, v = pisa_synth.random_qkv(700, 1, 1024, 128, dtype="bf16")
    run_attn(q, k, v, 64, 4, 1, "bf16", "recompute_tc")
    pisa.pisa_poll_device_status()


# ---------------------------------------------------------------------------
# the PISA hybrid path (global H-bar): GPU vs the oracle's hybrid form
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("Kfrac", [0.0, 0.25, 1.0])
def test_hybrid_small(d, B, order, Kfrac):
    L = 2048
    nblk = L // B
    K = int(round(Kfrac * nblk))
    q, k, v = pisa_synth.random_qkv(800 + d + B + order, 2, L, d, scale=2.0, dtype="bf16")
    got = run_attn(q, k, v, B, K, order, "bf16", "hybrid_tc")
    ref = oracle.pisa_hybrid(q, k, v, B, K, order)
    m = parity.check(got, ref, "bf16")
    assert m["rel_l2"] <= 5e-3, m


@pytest.mark.parametrize("case", ["ragged", "clustered", "sharp"])
def test_hybrid_edge_cases(case):
    d, B, L, K = 128, 64, 1152, 4
    scale = 8.0 if case == "sharp" else 2.0
    if case == "clustered":
        w = pisa_synth.workloads()["c2"].with_(heads=2, L=2048, n_centres=32, d=128)
        q, k, v = pisa_synth.generate(w)
        L, K = 2048, 4
    else:
        q, k, v = pisa_synth.random_qkv(850 + len(case), 2, L, d, scale=scale, dtype="bf16")
    got = run_attn(q, k, v, B, K, 1, "bf16", "hybrid_tc")
    ref = oracle.pisa_hybrid(q, k, v, B, K, 1)
    parity.check(got, ref, "bf16", case)


@pytest.mark.parametrize("name,per_head,nheads", [("c3", 2, 8), ("c4", 1, 4)] + [
    (f"c5_L{L}_s{sp}", 2, 8) for L in (4608, 16896) for sp in (50, 75, 90, 95)])
def test_hybrid_full_size_sampled(name, per_head, nheads):
    w, (q, k, v) = workload(name)
    got = run_attn(q, k, v, w.B, w.K, 1, w.dtype, "hybrid_tc")
    heads = list(np.random.default_rng(9).choice(w.BH, nheads, replace=False))
    tiles = sample_tiles(w.BH, w.nblk, per_head, seed=13, heads=heads)
    ref = oracle.pisa_hybrid(q, k, v, w.B, w.K, 1, tiles=tiles)
    parity.check(rows_of(got, tiles, w.B), ref, w.dtype, name)


# ---------------------------------------------------------------------------
# PWT's diagonal + pooled w (order 2, PISA_FLAG_POOLED_W)
# ---------------------------------------------------------------------------

def run_attn_w(q, k, v, B, K, order, dt, path, w_mode, gate=True):
    out = pisa.pisa_attention(dev(q, dt), dev(k, dt), dev(v, dt), B, K, order, gate=gate, path=path, w_mode=w_mode)
    pisa.pisa_poll_device_status()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("path", ["recompute_tc", "stats", "hybrid_tc", "stats_tc"])
@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (128, 128)])
@pytest.mark.parametrize("gate", [True, False])
def test_pooled_w_small(path, d, B, gate):
    L = 2048
    K = (L // B) // 4
    q, k, v = pisa_synth.random_qkv(900 + d + B, 2, L, d, scale=2.0, dtype="bf16")
    got = run_attn_w(q, k, v, B, K, 2, "bf16", path, "pooled", gate)
    ref = oracle.pisa_attention_ex(q, k, v, B, K, 2, gate=gate, hybrid=(path == "hybrid_tc"), w_pooled=True)
    m = parity.check(got, ref, "bf16")
    assert m["rel_l2"] <= 5e-3, m


def test_pooled_w_fp32_statistics_path():
    q, k, v = pisa_synth.random_qkv(950, 2, 1024, 64, scale=2.0, dtype="f32")
    got = run_attn_w(q, k, v, 64, 4, 2, "f32", "stats", "pooled")
    ref = oracle.pisa_attention_ex(q, k, v, 64, 4, 2, w_pooled=True)
    parity.check(got, ref, "f32")


def test_hybrid_order2_needs_pooled_w():
    q, k, v = pisa_synth.random_qkv(951, 1, 1024, 64, dtype="bf16")
    with pytest.raises(pisa.PisaError):
        run_attn_w(q, k, v, 64, 4, 2, "bf16", "hybrid_tc", "exact")


@pytest.mark.parametrize("path", ["recompute_tc", "hybrid_tc"])
def test_pooled_w_full_size_c2(path):
    w, (q, k, v) = workload("c2o2")
    got = run_attn_w(q, k, v, w.B, w.K, 2, w.dtype, path, "pooled")
    tiles = sample_tiles(w.BH, w.nblk, 4, seed=17, heads=[0, 5, 11])
    ref = oracle.pisa_attention_ex(q, k, v, w.B, w.K, 2, hybrid=(path == "hybrid_tc"), w_pooled=True, tiles=tiles)
    parity.check(rows_of(got, tiles, w.B), ref, w.dtype, path)


def test_host_entry_point_with_routing_matches_device_call():
    q, k, v = pisa_synth.random_qkv(77, 6, 1024, 128, scale=2.0, dtype="bf16")
    B, K = 64, 4
    dq, dk, dv = (dev(x, "bf16") for x in (q, k, v))
    want = pisa.pisa_attention(dq, dk, dv, B, K, 1, route="cov")
    hq, hk, hv = (t.cpu().pin_memory() for t in (dq, dk, dv))
    ho = torch.empty_like(hq).pin_memory()
    plan = pisa.HostPlan(hq, B, K, 1, chunk_heads=4)
    pisa.pisa_attention_host(hq, hk, hv, ho, plan, route="cov")
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    assert torch.equal(ho, want.cpu())


def test_host_entry_point_matches_device_call():
    # pisa_attention_host runs pisa_attention_ex per chunk of heads from pinned
    # host memory; heads are independent, so the result equals the device call.
    q, k, v = pisa_synth.random_qkv(990, 7, 2048, 128, scale=2.0, dtype="bf16")
    qt, kt, vt = (torch.from_numpy(x).to(torch.bfloat16) for x in (q, k, v))
    ref = pisa.pisa_attention(qt.cuda(), kt.cuda(), vt.cuda(), 64, 6, 1).cpu()
    hq, hk, hv = (x.pin_memory() for x in (qt, kt, vt))
    ho = torch.empty_like(hq).pin_memory()
    plan = pisa.HostPlan(hq, 64, 6, 1, chunk_heads=3)  # 3 + 3 + 1: a ragged last chunk
    pisa.pisa_attention_host(hq, hk, hv, ho, plan)
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    assert torch.equal(ho, ref)


# ---------------------------------------------------------------------------
# the largest block count the C ABI accepts: L / B = 4096
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", ["recompute_tc", "hybrid_tc"])
def test_maximum_block_count(path):
    # L = 4096 blocks x 64 tokens, d = 64, one head, 10 % of the blocks kept: score rows of 4096,
    # the top-K's scan branch and 128 mask words per row, bit-exact; sampled output tiles within
    # the bf16 tolerance
    B, d, K = 64, 64, 410
    L = 4096 * B
    q, k, v = pisa_synth.random_qkv(1900, 1, L, d, scale=2.0, dtype="bf16")
    st = pisa.pisa_centroids(dev(k, "bf16"), B)
    idx, mask = pisa.pisa_select(dev(q, "bf16"), st, K)
    torch.cuda.synchronize()
    ridx, rmask, _ = oracle.select(q, k, B, K)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(mask.cpu().numpy().view(np.uint32), rmask)
    got = run_attn(q, k, v, B, K, 1, "bf16", path)
    tiles = sample_tiles(1, L // B, 8, seed=13)
    ref = oracle.pisa_attention_ex(q, k, v, B, K, 1, hybrid=(path == "hybrid_tc"), tiles=tiles)
    parity.check(rows_of(got, tiles, B), ref, "bf16", path)


# ---------------------------------------------------------------------------
# numerics of the token form: the FMA-pipe exponential and w at a large offset
# ---------------------------------------------------------------------------

def test_ex2_fma_against_exact_powers_of_two():
    # the FMA-pipe 2^x the softmax uses for part of its exponentials: relative error within
    # the fitted 7.5e-5 (plus fp32 rounding) on [-125, 64], exactly 0 at and below -125
    xs = np.concatenate([np.linspace(-124.999, 63.999, 1 << 20), np.arange(-124, 64, 0.5),
                         [-125.0, -125.5, -200.0, -np.inf]]).astype(np.float32)
    y = pisa.pisa_selftest_ex2(torch.from_numpy(xs).cuda(), "fma").cpu().numpy()
    live = xs > -125.0
    exact = np.exp2(xs[live].astype(np.float64))
    rel = np.abs(y[live] - exact) / exact
    assert rel.max() <= 7.5e-5 + 2.0 ** -23, float(rel.max())
    assert np.all(y[~live] == 0.0)
    # the special-function unit's ex2.approx, for comparison: a few ulp on the same range
    z = pisa.pisa_selftest_ex2(torch.from_numpy(xs[live]).cuda(), "sfu").cpu().numpy()
    assert (np.abs(z - exact) / exact).max() <= 2.0 ** -20


@pytest.mark.parametrize("path", ["recompute_tc", "stats"])
def test_order2_with_a_large_common_logit_offset(path):
    # Every logit is about 300 (a shared channel) with a spread of about 1 inside each block, so
    # that w = (1/2B) sum_n (x_n - s-bar)^2 is O(1) while E[x^2] is about 9e4: a one-pass
    # variance in fp32 would lose w to cancellation.  The gate stays open (w < ln B).
    rng = np.random.default_rng(2024)
    BH, L, d, B, K = 2, 1024, 64, 64, 4
    q = np.empty((BH, L, d), np.float32)
    k = np.empty((BH, L, d), np.float32)
    q[..., 0] = 17.0
    k[..., 0] = 17.625  # 17 * 17.625 = 299.625, exact in bf16 products
    q[..., 1:] = 0.35 * rng.standard_normal((BH, L, d - 1))
    k[..., 1:] = 0.35 * rng.standard_normal((BH, L, d - 1))
    v = rng.standard_normal((BH, L, d)).astype(np.float32)
    q, k, v = (pisa_synth.round_bf16(x) for x in (q, k, v))
    got = run_attn(q, k, v, B, K, 2, "bf16", path)
    ref = oracle.pisa_attention(q, k, v, B, K, 2)
    parity.check(got, ref, "bf16", path)
    # w matters here: the result differs from order 1 by far more than the tolerance
    assert rel_l2(ref, oracle.pisa_attention(q, k, v, B, K, 1)) > 5e-2


# ---------------------------------------------------------------------------
# the statistics form on the tensor cores (PISA_PATH_STATS_TC): blocks selected
# by any tile of a 256-row CTA in the token form, every other block through the
# H_j contraction
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("Kfrac", [0.0, 0.1, 0.25, 0.5, 1.0])
def test_stats_tc_small(d, B, Kfrac):
    # K = 0: only the H_j contraction; K = all: only the union tiles; in between, both phases
    # with random selections (unions of different sizes, an odd number of contraction blocks
    # for d = 64, which pairs them)
    L = 2048
    nblk = L // B
    K = int(round(Kfrac * nblk))
    q, k, v = pisa_synth.random_qkv(1000 + d + B, 2, L, d, scale=2.0, dtype="bf16")
    got = run_attn(q, k, v, B, K, 1, "bf16", "stats_tc")
    ref = oracle.pisa_attention(q, k, v, B, K, 1)
    m = parity.check(got, ref, "bf16")
    assert m["rel_l2"] <= 5e-3, m


@pytest.mark.parametrize("case", ["ragged", "batched", "sharp", "clustered", "single_block", "max_raise"])
def test_stats_tc_edge_cases(case):
    d, B, L, BH, K, scale = 128, 128, 1024, 2, 2, 2.0
    batch = 1
    if case == "ragged":
        L = 1152  # 4.5 CTAs of 256 rows
        B = 64
    elif case == "batched":
        batch, BH = 2, 6
    elif case == "sharp":
        scale = 8.0  # large logits: the running max is raised in both phases
    elif case == "single_block":
        L, B, K = 128, 128, 0  # one block, one CTA with one live M tile
    if case == "clustered":
        w = pisa_synth.workloads()["c2"].with_(heads=2, L=4096)
        q, k, v = pisa_synth.generate(w)
        d, B, K = w.d, w.B, w.K
    else:
        q, k, v = pisa_synth.random_qkv(1100 + len(case), BH, L, d, scale=scale, dtype="bf16")
    if case == "max_raise":
        # the largest logits sit in the last blocks, which only the contraction phase reaches
        q[..., 0] = 2.0
        k[:, -2 * B:, 0] += 6.0
        q, k = pisa_synth.round_bf16(q), pisa_synth.round_bf16(k)
        K = 0
    qt, kt, vt = (dev(x, "bf16") for x in (q, k, v))
    if batch > 1:
        qt, kt, vt = (x.view(batch, BH // batch, L, d) for x in (qt, kt, vt))
    got = pisa.pisa_attention(qt, kt, vt, B, K, 1, path="stats_tc").float().cpu().numpy().reshape(q.shape)
    pisa.pisa_poll_device_status()
    parity.check(got, oracle.pisa_attention(q, k, v, B, K, 1), "bf16", case)


def test_stats_tc_agrees_with_the_token_form():
    # the two tensor-core associations of the same first-order term, on the same inputs
    q, k, v = pisa_synth.random_qkv(1200, 3, 4096, 64, scale=2.0, dtype="bf16")
    a = run_attn(q, k, v, 64, 12, 1, "bf16", "stats_tc")
    b = run_attn(q, k, v, 64, 12, 1, "bf16", "recompute_tc")
    parity.check(a, b, "bf16", "stats_tc vs recompute_tc")


def test_auto_runs_the_statistics_form_at_the_hunyuan_and_clustered_shapes():
    assert pisa.pisa_resolve_path(1, 24, 118784, 128, 128, 93, 1, torch.bfloat16) == "stats_tc"
    assert pisa.pisa_resolve_path(1, 12, 8192, 64, 64, 16, 1, torch.bfloat16) == "stats_tc"
    w = pisa_synth.workloads()["c2"].with_(heads=3)
    q, k, v = pisa_synth.generate(w)
    auto = run_attn(q, k, v, w.B, w.K, 1, w.dtype, "auto")
    assert np.array_equal(auto, run_attn(q, k, v, w.B, w.K, 1, w.dtype, "stats_tc"))


def test_hybrid_is_reproducible():
    # H-bar is summed over the prepare kernel's chunks in a fixed order (no atomics), so two
    # calls on the same inputs give the same output bit for bit
    q, k, v = pisa_synth.random_qkv(870, 6, 8192, 128, scale=2.0, dtype="bf16")
    a = run_attn(q, k, v, 64, 16, 1, "bf16", "hybrid_tc")
    for _ in range(2):
        assert np.array_equal(a, run_attn(q, k, v, 64, 16, 1, "bf16", "hybrid_tc"))
