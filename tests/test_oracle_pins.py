"""Pins for the CPU oracle: checks against facts the pages and the mathematics fix.

None of these tests compares the oracle with itself.  Each pin reaches the
expected value through a different route: a library routine (torch fp64
softmax), a closed form, a special case that reduces to exact attention, an
invariant, the error bound of the PISA paper's Appendix C, brute force per
token, or a hand-built fixture.  A plausible mistake in the oracle (a dropped
term, a wrong sign, a transposed statistic, a wrong normalisation, a wrong tie
rule, a clamp instead of the gate) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import pisa_synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def torch_dense(q, k, v):
    """softmax(q k^T) v in fp64 through torch (PISA paper section 3.1, Eq. 1)."""
    qt, kt, vt = (torch.from_numpy(np.asarray(x, np.float64)) for x in (q, k, v))
    return torch.softmax(qt @ kt.transpose(-1, -2), dim=-1).matmul(vt).numpy()


def torch_lse(q, k):
    qt, kt = (torch.from_numpy(np.asarray(x, np.float64)) for x in (q, k))
    return torch.logsumexp(qt @ kt.transpose(-1, -2), dim=-1).numpy()


def small(seed, BH=2, L=256, d=16, scale=1.0):
    return pisa_synth.random_qkv(seed, BH, L, d, scale=scale)


# ----------------------------------------------------------------------------
# exact special cases
# ----------------------------------------------------------------------------

def test_dense_oracle_matches_torch():
    q, k, v = small(1, L=128, d=8, scale=3.0)
    np.testing.assert_allclose(oracle.dense_attention(q, k, v), torch_dense(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("order", [0, 1, 2])
def test_all_blocks_selected_equals_dense(order):
    # With U empty the method is exact softmax attention (PISA section 3.2, D_t with U = {}).
    q, k, v = small(2, L=256, d=16, scale=2.0)
    B = 16
    o = oracle.pisa_attention(q, k, v, B, 256 // B, order=order)
    np.testing.assert_allclose(o, torch_dense(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("K", [0, 3, 17])
@pytest.mark.parametrize("order", [0, 1, 2])
def test_block_size_one_is_exact(K, order):
    # B = 1: every centroid is its key, every deviation is zero.
    q, k, v = small(3, L=32, d=8, scale=2.0)
    o = oracle.pisa_attention(q, k, v, 1, K, order=order)
    np.testing.assert_allclose(o, torch_dense(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("order", [0, 1, 2])
def test_identical_keys_per_block_is_exact(order):
    # K = 0 with equal keys inside each block: the Taylor expansion is exact.
    q, k, v = small(4, L=128, d=8, scale=2.0)
    B = 16
    k = np.repeat(k[:, ::B, :], B, axis=1).copy()
    o = oracle.pisa_attention(q, k, v, B, 0, order=order)
    np.testing.assert_allclose(o, torch_dense(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("order", [0, 1, 2])
@pytest.mark.parametrize("K", [0, 2, 8])
def test_zero_queries_give_mean_value(order, K):
    # q = 0: every logit is 0 and every weight (exact or virtual token) is uniform.
    _, k, v = small(5, L=128, d=8)
    q = np.zeros_like(k)
    o = oracle.pisa_attention(q, k, v, 16, K, order=order)
    np.testing.assert_allclose(o, np.broadcast_to(v.astype(np.float64).mean(axis=1, keepdims=True), o.shape), atol=1e-13)


def test_constant_values_per_block_remove_first_order():
    # H_j = sum_n v_n (k_n - kbar_j)^T vanishes when v is constant in the block.
    q, k, v = small(6, L=128, d=8, scale=2.0)
    B = 16
    v = np.repeat(v[:, ::B, :], B, axis=1).copy()
    o1 = oracle.pisa_attention(q, k, v, B, 2, order=1)
    o0 = oracle.pisa_attention(q, k, v, B, 2, order=0)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------
# brute force per token (no block statistics)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("order", [0, 1, 2])
@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("B,d,K", [(16, 16, 3), (32, 8, 1), (8, 32, 10), (64, 16, 0)])
def test_statistics_form_equals_token_form(order, gate, B, d, K):
    q, k, v = small(7 + B + d, L=256, d=d, scale=2.0)
    o = oracle.pisa_attention(q, k, v, B, K, order=order, gate=gate)
    ob = oracle.pisa_bruteforce(q, k, v, B, K, order=order, gate=gate)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# block statistics: invariants and closed forms
# ----------------------------------------------------------------------------

def test_statistics_invariants():
    q, k, v = small(8, BH=1, L=128, d=16, scale=1.0)
    B = 8  # B < d, so rank(H_j) <= B - 1 < d is visible
    kbar, vsum, H, C = oracle.block_stats(k, v, B, order=2)
    kb = k[0].reshape(-1, B, 16).astype(np.float64)
    vb = v[0].reshape(-1, B, 16).astype(np.float64)
    np.testing.assert_allclose(kbar[0], kb.mean(axis=1), atol=1e-14)
    np.testing.assert_allclose(vsum[0], vb.sum(axis=1), atol=1e-13)
    for j in range(kb.shape[0]):
        dev = kb[j] - kb[j].mean(axis=0)
        # H_j q = sum_n v_n (q . (k_n - kbar_j)): pins the orientation (rows = value channel)
        qq = q[0, j].astype(np.float64)
        np.testing.assert_allclose(H[0, j] @ qq, (vb[j] * (dev @ qq)[:, None]).sum(axis=0), atol=1e-12)
        # the deviations sum to zero, so H_j annihilates nothing in general but H_j has rank <= B - 1
        sv = np.linalg.svd(H[0, j], compute_uv=False)
        assert sv[B - 1] < 1e-10 * sv[0]
        # trace C_j = (1/B) sum_n |k_n - kbar|^2 = (1/2B^2) sum_{n,n'} |k_n - k_n'|^2
        pair = ((kb[j][:, None, :] - kb[j][None, :, :]) ** 2).sum()
        assert abs(np.trace(C[0, j]) - pair / (2 * B * B)) < 1e-12
        # C_j is symmetric positive semi-definite
        np.testing.assert_allclose(C[0, j], C[0, j].T, atol=0)
        assert np.linalg.eigvalsh(C[0, j]).min() > -1e-12


def test_statistics_vanish_for_identical_keys_and_constant_values():
    _, k, v = small(9, BH=1, L=64, d=8)
    B = 16
    k = np.repeat(k[:, ::B, :], B, axis=1).copy()
    _, _, H, C = oracle.block_stats(k, v, B, order=2)
    assert np.abs(H).max() == 0.0 and np.abs(C).max() == 0.0
    _, k2, _ = small(10, BH=1, L=64, d=8)
    v2 = np.repeat(v[:, ::B, :], B, axis=1).copy()
    _, _, H2, _ = oracle.block_stats(k2, v2, B, order=1)
    assert np.abs(H2).max() < 1e-13


def test_second_order_two_point_block_closed_form():
    # Keys kbar + a (B/2 tokens) and kbar - a (B/2 tokens): C_j = a a^T, so
    # w = 1/2 (q.a)^2 exactly, and the single virtual token has mass B e^{q.kbar + w}
    # ("Sparse Linear Attention" blog, PWT section).  The true mass is
    # B e^{q.kbar} cosh(q.a), which e^{w} approaches more closely than 1 does.
    rng = np.random.default_rng(11)
    B, d = 16, 8
    kbar = rng.integers(-2, 3, d).astype(np.float32) / 4
    a = rng.integers(-2, 3, d).astype(np.float32) / 8
    k = np.concatenate([np.tile(kbar + a, (B // 2, 1)), np.tile(kbar - a, (B // 2, 1))])[None]
    q = (rng.integers(-3, 4, (1, B, d)).astype(np.float32) / 8)
    v = rng.standard_normal((1, B, d)).astype(np.float32)
    _, lse2 = oracle.pisa_attention(q, k, v, B, 0, order=2, gate=False, want_lse=True)
    _, lse1 = oracle.pisa_attention(q, k, v, B, 0, order=1, want_lse=True)
    qa = q[0].astype(np.float64) @ a.astype(np.float64)
    qk = q[0].astype(np.float64) @ kbar.astype(np.float64)
    np.testing.assert_allclose(lse1[0], math.log(B) + qk, atol=1e-12)
    np.testing.assert_allclose(lse2[0], math.log(B) + qk + 0.5 * qa ** 2, atol=1e-12)
    true = np.log(B * np.exp(qk) * np.cosh(qa))
    assert np.all(np.abs(lse2[0] - true) <= np.abs(lse1[0] - true) + 1e-15)


def test_second_order_gate_zeroes_not_clamps():
    # Huge within-block spread: every w exceeds ln B, so the gated order-2 result
    # must equal order 1 exactly (a clamp at ln B would not).
    q, k, v = small(12, L=128, d=8, scale=1.0)
    B = 16
    k = k * np.float32(40.0)
    o1 = oracle.pisa_attention(q, k, v, B, 2, order=1)
    o2 = oracle.pisa_attention(q, k, v, B, 2, order=2, gate=True)
    o2n = oracle.pisa_attention(q, k, v, B, 2, order=2, gate=False)
    assert np.array_equal(o1, o2)
    assert not np.allclose(o1, o2n)


# ----------------------------------------------------------------------------
# denominators and the error bound (PISA paper, Appendix C)
# ----------------------------------------------------------------------------

def test_jensen_denominator_and_nonnegative_w():
    # B alpha_{t,j} <= sum_n exp(q k_{j,n}) (Appendix C), so the approximate
    # denominator never exceeds the dense one; w >= 0 so order 2 adds mass.
    q, k, v = small(13, L=256, d=16, scale=2.0)
    B = 16
    dense = torch_lse(q, k)
    _, l1 = oracle.pisa_attention(q, k, v, B, 4, order=1, want_lse=True)
    _, l0 = oracle.pisa_attention(q, k, v, B, 4, order=0, want_lse=True)
    _, l2 = oracle.pisa_attention(q, k, v, B, 4, order=2, gate=False, want_lse=True)
    assert np.all(l1 <= dense + 1e-12)
    np.testing.assert_array_equal(l0, l1)  # the first-order mass is exactly zero
    assert np.all(l2 >= l1 - 1e-12)


def _bound_terms(q, k, v, B, K):
    """Per row: C_v e^{eta} S_2 / D-hat for the per-block first-order form."""
    q64, k64, v64 = (np.asarray(x, np.float64) for x in (q, k, v))
    BH, L, d = q.shape
    nblk = L // B
    _, mask, _ = oracle.select(q, k, B, K)
    bound = np.zeros((BH, L))
    for bh in range(BH):
        cv = np.linalg.norm(v64[bh], axis=1).max()
        kb = k64[bh].reshape(nblk, B, d)
        kbar = kb.mean(axis=1)
        for i in range(nblk):
            sel = np.array([(mask[bh, i, j // 32] >> (j % 32)) & 1 for j in range(nblk)], bool)
            qt = q64[bh, i * B:(i + 1) * B]                       # [B, d]
            x = np.einsum("td,jnd->tjn", qt, kb)                   # logits
            sbar = qt @ kbar.T                                     # [B, nblk]
            delta = x - sbar[:, :, None]
            alpha = np.exp(sbar)
            dhat = (np.exp(x) * sel[None, :, None]).sum(axis=(1, 2)) + (B * alpha * ~sel[None, :]).sum(axis=1)
            s2 = (alpha[:, ~sel] * (delta[:, ~sel, :] ** 2).sum(axis=2)).sum(axis=1)
            eta = np.abs(delta[:, ~sel, :]).max(axis=(1, 2)) if (~sel).any() else np.zeros(B)
            bound[bh, i * B:(i + 1) * B] = cv * np.exp(eta) * s2 / dhat
    return bound


def test_taylor_error_bound_appendix_c():
    # ||o-hat - o*|| <= C_v e^{eta} S_2 / D-hat for block-wise H_j (Appendix C);
    # the zeroth-order variant, which drops H_j q, must break it somewhere at
    # small eta (its error is first order in eta).
    B, K = 16, 4
    for scale in (1.0, 0.25, 0.02):
        q, k, v = small(14, BH=2, L=256, d=16, scale=scale)
        bound = _bound_terms(q, k, v, B, K)
        dense = torch_dense(q, k, v)
        err1 = np.linalg.norm(oracle.pisa_attention(q, k, v, B, K, order=1) - dense, axis=-1)
        assert np.all(err1 <= bound * (1 + 1e-9) + 1e-15)
        if scale == 0.02:
            err0 = np.linalg.norm(oracle.pisa_attention(q, k, v, B, K, order=0) - dense, axis=-1)
            assert np.any(err0 > bound)


# ----------------------------------------------------------------------------
# canonical fp32 selection
# ----------------------------------------------------------------------------

def np_tree_sum(a, axis):
    """The canonical pairwise tree in numpy float32 (a[i] += a[i + h], h = n/2 .. 1)."""
    a = np.moveaxis(np.asarray(a, np.float32), axis, 0).copy()
    n = a.shape[0]
    while n > 1:
        h = n // 2
        a[:h] = a[:h] + a[h:n]
        n = h
    return a[0]


def np_select(q, k, B, K):
    BH, L, d = q.shape
    nblk = L // B
    inv = np.float32(1.0 / B)
    idx = np.zeros((BH, nblk, K), np.int32)
    scores = np.zeros((BH, nblk, nblk), np.float32)
    for bh in range(BH):
        qbar = np_tree_sum(q[bh].reshape(nblk, B, d), 1) * inv
        kbar = np_tree_sum(k[bh].reshape(nblk, B, d), 1) * inv
        prod = qbar[:, None, :] * kbar[None, :, :]
        s = np_tree_sum(prod, 2)
        scores[bh] = s
        for i in range(nblk):
            order = np.lexsort((np.arange(nblk), -s[i].astype(np.float64)))
            idx[bh, i] = np.sort(order[:K])
    return idx, scores


@pytest.mark.parametrize("B,d,K,dtype", [(16, 16, 5, "f32"), (64, 64, 4, "f32"), (32, 128, 7, "bf16"),
                                         (8, 8, 0, "f32"), (8, 8, 32, "f32")])
def test_selection_matches_numpy_restatement_bitwise(B, d, K, dtype):
    L = 256
    q, k, _ = pisa_synth.random_qkv(15 + B, 2, L, d, scale=4.0, dtype=dtype)
    idx, mask, scores = oracle.select(q, k, B, K, want_scores=True)
    idx_np, scores_np = np_select(q, k, B, K)
    assert np.array_equal(scores.view(np.uint32), scores_np.view(np.uint32))
    assert np.array_equal(idx, idx_np)
    nblk = L // B
    for bh in range(2):
        for i in range(nblk):
            bits = [j for j in range(nblk) if (mask[bh, i, j // 32] >> (j % 32)) & 1]
            assert bits == list(idx[bh, i])


def test_selection_tie_rule_golden():
    with open(os.path.join(GOLDEN, "tie_break.json")) as f:
        g = json.load(f)
    q = np.asarray(g["q"], np.float32)[None]
    k = np.asarray(g["k"], np.float32)[None]
    _, _, scores = oracle.select(q, k, g["B"], 1, want_scores=True)
    np.testing.assert_array_equal(scores[0], np.asarray(g["scores_by_hand"], np.float32))
    for K, want in g["expected_idx"].items():
        idx, _, _ = oracle.select(q, k, g["B"], int(K))
        np.testing.assert_array_equal(idx[0], np.asarray(want, np.int32))


def test_selection_agrees_with_fp64_ranking_away_from_ties():
    q, k, _ = pisa_synth.random_qkv(16, 2, 512, 32, scale=4.0)
    B, K = 16, 6
    idx, _, _ = oracle.select(q, k, B, K)
    q64, k64 = q.astype(np.float64), k.astype(np.float64)
    nblk = 512 // B
    for bh in range(2):
        s = q64[bh].reshape(nblk, B, -1).mean(1) @ k64[bh].reshape(nblk, B, -1).mean(1).T
        for i in range(nblk):
            srt = np.sort(s[i])[::-1]
            gap = srt[K - 1] - srt[K]
            if gap > 1e-4 * max(1.0, abs(srt[K])):
                want = np.sort(np.argsort(-s[i], kind="stable")[:K])
                assert np.array_equal(idx[bh, i], want)


def test_oracle_rejects_undefined_shapes():
    q, k, v = small(17, L=96, d=8)
    with pytest.raises(ValueError):
        oracle.select(q, k, 12, 2)        # B not a power of two
    with pytest.raises(ValueError):
        oracle.pisa_attention(q, k, v, 64, 1)  # L % B != 0
    with pytest.raises(ValueError):
        oracle.pisa_attention(q, k, v, 16, 7)  # K > nblk


def test_canonical_centroids_match_numpy_restatement():
    _, k, _ = pisa_synth.random_qkv(18, 2, 512, 64, dtype="bf16")
    for B in (16, 64, 128):
        c = oracle.centroids_f32(k, B)
        ref = np_tree_sum(k.reshape(2, 512 // B, B, 64), 2) * np.float32(1.0 / B)
        assert np.array_equal(c.view(np.uint32), ref.view(np.uint32))


# ----------------------------------------------------------------------------
# the PISA hybrid (global H-bar), "Sparse Linear Attention" blog and PISA
# paper section 3.3 / Appendix C
# ----------------------------------------------------------------------------

def test_hybrid_equals_per_block_when_every_block_has_the_same_statistic():
    # Shifting a block's keys by a constant leaves its deviations unchanged, so
    # blocks built as (base keys + shift_j, base values) all share one H_j;
    # then H-bar = H_j and the hybrid is the per-block first-order form.
    rng = np.random.default_rng(19)
    B, d, nblk = 16, 8, 16
    # dyadic values: every shifted key is exact in fp32, so the deviations agree bit for bit
    kb = (rng.integers(-16, 17, (B, d)) / 8.0).astype(np.float32)
    vb = rng.standard_normal((B, d)).astype(np.float32)
    shifts = (rng.integers(-4, 5, (nblk, 1, d)) / 4.0).astype(np.float32)
    k = (kb[None] + shifts).reshape(1, nblk * B, d).astype(np.float32)
    v = np.tile(vb, (nblk, 1))[None].astype(np.float32)
    q = (rng.standard_normal((1, nblk * B, d)) * 0.5).astype(np.float32)
    np.testing.assert_allclose(oracle.pisa_hybrid(q, k, v, B, 3, 1), oracle.pisa_attention(q, k, v, B, 3, 1),
                               rtol=0, atol=1e-12)


def test_hybrid_numerator_differs_by_the_appendix_c_residual():
    # N_hybrid - N_per-block = sum_U alpha_tj (H-bar - H_j) q_t  (= -q R_t in
    # Appendix C) while the denominators agree, so
    # (o_hybrid - o_per-block) * D-hat = sum_U alpha_tj (H-bar - H_j) q_t.
    q, k, v = small(20, BH=1, L=256, d=16, scale=1.0)
    B, K = 16, 3
    oh, lh = oracle.pisa_hybrid(q, k, v, B, K, 1, want_lse=True)
    op, lp = oracle.pisa_attention(q, k, v, B, K, 1, want_lse=True)
    np.testing.assert_allclose(lh, lp, rtol=0, atol=1e-12)
    q64, k64, v64 = (np.asarray(x[0], np.float64) for x in (q, k, v))
    nblk = 256 // B
    kb = k64.reshape(nblk, B, 16)
    vb = v64.reshape(nblk, B, 16)
    H = np.einsum("jna,jnb->jab", vb, kb - kb.mean(axis=1, keepdims=True))
    Hbar = H.mean(axis=0)
    _, mask, _ = oracle.select(q, k, B, K)
    for i in range(nblk):
        sel = np.array([(mask[0, i, j // 32] >> (j % 32)) & 1 for j in range(nblk)], bool)
        for m in range(B):
            t = i * B + m
            alpha = np.exp(q64[t] @ kb.mean(axis=1).T)                 # unshifted e^{q.kbar_j}
            resid = sum(alpha[j] * ((Hbar - H[j]) @ q64[t]) for j in range(nblk) if not sel[j])
            np.testing.assert_allclose((oh[0, t] - op[0, t]) * np.exp(lh[0, t]), resid, rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("order", [0, 1, 2])
def test_hybrid_special_cases(order):
    q, k, v = small(21, L=256, d=16, scale=2.0)
    B = 16
    np.testing.assert_allclose(oracle.pisa_hybrid(q, k, v, B, 16, order), torch_dense(q, k, v), rtol=0, atol=1e-12)
    if order == 0:
        np.testing.assert_array_equal(oracle.pisa_hybrid(q, k, v, B, 4, 0), oracle.pisa_attention(q, k, v, B, 4, 0))


# ----------------------------------------------------------------------------
# PWT's diagonal + pooled second-order correction ("Sparse Linear Attention"
# blog, PWT section): w_ij = 1/2 sum_c mean_{t in tile i}(q_tc^2) sigma^2_jc
# ----------------------------------------------------------------------------

def test_pooled_w_equals_exact_w_for_constant_tile_queries_and_diagonal_covariance():
    # Keys that vary in one channel only make C_j diagonal; queries that are the
    # same on every row of a tile make mean(q^2) = q^2.  Then the pooled
    # diagonal estimate equals the exact 1/2 q^T C_j q.
    rng = np.random.default_rng(22)
    B, d, nblk = 16, 8, 8
    L = B * nblk
    k = np.repeat(rng.standard_normal((1, nblk, 1, d)), B, axis=2).astype(np.float32)
    k[..., 0] += (rng.integers(-4, 5, (1, nblk, B)) / 4.0).astype(np.float32)
    k = k.reshape(1, L, d)
    q = np.repeat((rng.standard_normal((1, nblk, 1, d)) * 0.4).astype(np.float32), B, axis=2).reshape(1, L, d)
    v = rng.standard_normal((1, L, d)).astype(np.float32)
    for gate in (True, False):
        e = oracle.pisa_attention_ex(q, k, v, B, 2, 2, gate=gate)
        p = oracle.pisa_attention_ex(q, k, v, B, 2, 2, gate=gate, w_pooled=True)
        np.testing.assert_allclose(p, e, rtol=0, atol=1e-12)


def test_pooled_w_closed_form_and_square_before_mean():
    # One block (K = 0): log D_t = log B + q_t . kbar + w with one w for the tile,
    # w = 1/2 sum_c mean_t(q_tc^2) var_c(k).  Rows +a and -a have mean q = 0, so a
    # "square of the mean" pooling would give w = 0; the blog's pooling does not.
    rng = np.random.default_rng(23)
    B, d = 16, 8
    k = (rng.integers(-8, 9, (1, B, d)) / 8.0).astype(np.float32)
    a = (rng.integers(-4, 5, d) / 16.0).astype(np.float32)
    q = np.concatenate([np.tile(a, (B // 2, 1)), np.tile(-a, (B // 2, 1))])[None].astype(np.float32)
    v = rng.standard_normal((1, B, d)).astype(np.float32)
    _, lse = oracle.pisa_attention_ex(q, k, v, B, 0, 2, gate=False, w_pooled=True, want_lse=True)
    k64 = k[0].astype(np.float64)
    var = ((k64 - k64.mean(axis=0)) ** 2).mean(axis=0)
    q64 = q[0].astype(np.float64)
    w = 0.5 * ((q64 ** 2).mean(axis=0) * var).sum()
    assert w > 0
    np.testing.assert_allclose(lse[0], np.log(B) + q64 @ k64.mean(axis=0) + w, rtol=0, atol=1e-12)


def test_pooled_w_gate_and_other_orders():
    q, k, v = small(24, L=128, d=8, scale=1.0)
    B = 16
    k40 = k * np.float32(40.0)  # every pooled w exceeds ln B: the gate gives order 1 back
    np.testing.assert_array_equal(oracle.pisa_attention_ex(q, k40, v, B, 2, 2, w_pooled=True),
                                  oracle.pisa_attention(q, k40, v, B, 2, 1))
    # the pooled flag changes nothing below order 2
    np.testing.assert_array_equal(oracle.pisa_attention_ex(q, k, v, B, 2, 1, w_pooled=True),
                                  oracle.pisa_attention(q, k, v, B, 2, 1))


# --------------------------------------------------------------------------
# Covariance-aware routing (PISA paper, section 3.3 "Covariance-Aware Block
# Selection"; "Sparse Linear Attention" blog, PWT section: route by the block
# score plus the log of the norm of H_j).  Reading: bias_j = ln(||H_j||_F + eps)
# in a canonical fp32 procedure, added to the centroid score.
# --------------------------------------------------------------------------


def test_ln_f32_accuracy():
    # error budget: the fp32 ln 2 constant and the rounding of e ln 2 (2 x 2^-24 |e ln 2|),
    # the final add (2^-24 |ln x|), the series on [sqrt(1/2), sqrt(2)) (~1e-7 absolute)
    rng = np.random.default_rng(31)
    x = np.exp(rng.uniform(math.log(1e-6), math.log(1e30), 100000)).astype(np.float32)
    x = np.concatenate([x, (1.0 + rng.uniform(-0.3, 0.3, 20000)).astype(np.float32)])
    y = oracle.ln_f32(x).astype(np.float64)
    ref = np.log(x.astype(np.float64))
    assert np.all(np.abs(y - ref) <= 3 * 2.0 ** -24 * np.abs(ref) + 1.2e-7)


def test_ln_f32_exact_points():
    # ln 1 = 0 exactly; at x = 2^e the mantissa term vanishes and the result is fl(e * fl(ln 2))
    assert oracle.ln_f32(np.array([1.0], np.float32))[0] == 0.0
    es = np.arange(-19, 100, dtype=np.int64)
    x = np.ldexp(np.ones(es.shape), es).astype(np.float32)
    want = es.astype(np.float32) * np.float32(math.log(2.0))
    np.testing.assert_array_equal(oracle.ln_f32(x), want)


def test_route_bias_is_log_frobenius_norm_of_h():
    q, k, v = small(41, L=256, d=16, scale=1.0)
    B, eps = 16, 1e-6
    _, _, H, _ = oracle.block_stats(k, v, B, order=1)
    want = np.log(np.sqrt((H ** 2).sum(axis=(2, 3))) + eps)
    got = oracle.route_bias(k, v, B, eps)
    assert got.shape == want.shape and got.dtype == np.float32
    np.testing.assert_allclose(got, want, rtol=0, atol=2e-5)


def test_route_bias_of_a_constant_key_block_is_log_eps():
    # identical keys inside a block: k - kbar = 0 exactly, H_j = 0, bias = ln(eps)
    rng = np.random.default_rng(43)
    B, d, nblk = 16, 8, 4
    k = np.repeat(rng.integers(-8, 9, (1, nblk, 1, d)) / 8.0, B, axis=2).reshape(1, nblk * B, d).astype(np.float32)
    v = rng.standard_normal((1, nblk * B, d)).astype(np.float32)
    for eps in (1e-6, 0.5, 3.0):
        got = oracle.route_bias(k, v, B, eps)
        np.testing.assert_array_equal(got, np.full((1, nblk), oracle.ln_f32(np.array([eps], np.float32))[0]))
        np.testing.assert_allclose(got, math.log(np.float32(eps)), rtol=0, atol=1e-6)


def test_biased_selection_restated_in_numpy():
    # the bias enters as one fp32 add after the canonical score, then the same
    # total order (score descending, block index ascending)
    q, k, v = small(47, L=512, d=16, scale=1.0)
    B, K = 16, 7
    _, _, s = oracle.select(q, k, B, K, want_scores=True)
    bias = oracle.route_bias(k, v, B)
    idx, mask, sb = oracle.select(q, k, B, K, want_scores=True, bias=bias)
    s2 = (s + bias[:, None, :]).astype(np.float32)  # float32 + float32: one rounding
    np.testing.assert_array_equal(sb, s2)
    nblk = s.shape[-1]
    for bh in range(s.shape[0]):
        for i in range(nblk):
            order = sorted(range(nblk), key=lambda j: (-float(s2[bh, i, j]), j))
            np.testing.assert_array_equal(idx[bh, i], np.sort(order[:K]))


def test_routing_sends_a_heterogeneous_block_to_the_exact_branch():
    # two candidate blocks with (nearly) the same centroid score: block 1 has
    # identical keys (Taylor is exact there, bias ln eps), block 2 spreads its keys
    # (large H_j).  The plain score keeps block 1 (slightly higher); routing keeps block 2.
    B, d = 16, 8
    rng = np.random.default_rng(53)
    base = np.zeros(d, np.float32)
    base[0] = 1.0
    k = np.zeros((1, 4 * B, d), np.float32)
    k[0, 0:B] = -base                       # block 0: far away
    k[0, B:2 * B] = base * 1.01             # block 1: identical keys, score slightly higher
    spread = rng.choice([-2.0, 2.0], (B, d)).astype(np.float32)
    spread -= spread.mean(axis=0)
    k[0, 2 * B:3 * B] = base + spread       # block 2: same centroid direction, spread out
    k[0, 3 * B:4 * B] = -2 * base           # block 3: far away
    q = np.tile(base, (1, 4 * B, 1)).astype(np.float32)
    v = rng.standard_normal((1, 4 * B, d)).astype(np.float32)
    plain, _, _ = oracle.select(q, k, B, 1)
    routed, _, _ = oracle.select(q, k, B, 1, bias=oracle.route_bias(k, v, B))
    assert plain[0, 0, 0] == 1 and routed[0, 0, 0] == 2


def test_routed_attention_matches_dense_when_every_block_is_selected():
    q, k, v = small(59, L=256, d=16, scale=1.0)
    B = 16
    got = oracle.pisa_attention_ex(q, k, v, B, 256 // B, 1, route_eps=1e-6)
    np.testing.assert_allclose(got, oracle.dense_attention(q, k, v), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Gradients (the backward pass; the pages print no equations, the oracle's
# are derived from its forward with the selection held fixed)
# --------------------------------------------------------------------------


def _dyadic_qkv(seed, L, d):
    rng = np.random.default_rng(seed)
    return tuple((rng.integers(-64, 65, (1, L, d)) / 64.0).astype(np.float32) for _ in range(3))


@pytest.mark.parametrize("order,gate", [(0, True), (1, True), (2, False), (2, True)])
def test_backward_matches_central_differences(order, gate):
    # dyadic inputs and step 2^-10 keep every perturbed input exact in fp32; the
    # loss is sum(dO . o) in fp64; coordinates whose perturbation changes the
    # (fixed) selection are skipped
    L, d, B, K = 64, 4, 16, 2
    q, k, v = _dyadic_qkv(61 + order, L, d)
    q *= 2.0
    dO = _dyadic_qkv(67, L, d)[0]
    gq, gk, gv = oracle.pisa_backward(q, k, v, dO, B, K, order, gate)
    _, mask0, _ = oracle.select(q, k, B, K)
    h = 2.0 ** -10

    def loss(q_, k_, v_):
        return float((oracle.pisa_attention(q_, k_, v_, B, K, order, gate=gate) * dO).sum())

    rng = np.random.default_rng(5)
    checked = 0
    for name, x, g in (("q", q, gq), ("k", k, gk), ("v", v, gv)):
        for _ in range(20):
            idx = (0, int(rng.integers(L)), int(rng.integers(d)))
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            if name != "v" and not (np.array_equal(oracle.select(args_p[0], args_p[1], B, K)[1], mask0) and
                                    np.array_equal(oracle.select(args_m[0], args_m[1], B, K)[1], mask0)):
                continue
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) <= 2e-5 * max(1.0, abs(g[idx])), (name, idx, fd, g[idx])
            checked += 1
    assert checked >= 40


def test_backward_with_every_block_selected_is_the_dense_gradient():
    # K = all blocks: the method is dense softmax attention; its gradient from
    # torch autograd in fp64 (a library, independent of the derivation)
    L, d, B = 64, 8, 16
    q, k, v = small(71, BH=2, L=L, d=d, scale=1.5)
    dO = small(72, BH=2, L=L, d=d)[0]
    gq, gk, gv = oracle.pisa_backward(q, k, v, dO, B, L // B, 1)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = torch.softmax(tq @ tk.transpose(1, 2), dim=-1) @ tv
    (o * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    for g, t in ((gq, tq), (gk, tk), (gv, tv)):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=0, atol=1e-11)


def test_backward_order0_identical_keys_is_exact_attention_gradient_for_v():
    # identical keys in every block: every unselected block's virtual token is
    # exact, so the output equals dense attention and dv does too (dv is linear
    # in the weights, which match exactly)
    L, d, B, K = 64, 8, 16, 1
    rng = np.random.default_rng(73)
    k = np.repeat(rng.standard_normal((1, L // B, 1, d)), B, axis=2).reshape(1, L, d).astype(np.float32)
    q = rng.standard_normal((1, L, d)).astype(np.float32)
    v = rng.standard_normal((1, L, d)).astype(np.float32)
    dO = rng.standard_normal((1, L, d)).astype(np.float32)
    _, _, gv = oracle.pisa_backward(q, k, v, dO, B, K, 0)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = torch.softmax(tq @ tk.transpose(1, 2), dim=-1) @ tv
    (o * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    np.testing.assert_allclose(gv, tv.grad.numpy(), rtol=0, atol=1e-11)


def test_backward_with_routing_matches_central_differences():
    # covariance-aware selection (PISA paper section 3.3; PWT section of the
    # "Sparse Linear Attention" blog): the routing only picks the blocks, so the
    # gradient is the same formula on the routed selection; coordinates whose
    # perturbation changes the routed selection are skipped
    L, d, B, K = 64, 4, 16, 2
    eps = 1e-6
    q, k, v = _dyadic_qkv(81, L, d)
    q *= 2.0
    v[:, 16:32] *= 4.0  # a block with a large ||H_j||: routing changes the selection
    dO = _dyadic_qkv(83, L, d)[0]
    gq, gk, gv = oracle.pisa_backward(q, k, v, dO, B, K, 1, True, route_eps=eps)

    def rmask(q_, k_, v_):
        return oracle.select(q_, k_, B, K, bias=oracle.route_bias(k_, v_, B, eps))[1]

    mask0 = rmask(q, k, v)
    assert not np.array_equal(mask0, oracle.select(q, k, B, K)[1])
    # the plain backward on other blocks differs: routing reaches the gradient
    assert oracle.rel_l2(oracle.pisa_backward(q, k, v, dO, B, K, 1)[0], gq) > 1e-3
    h = 2.0 ** -10

    def loss(q_, k_, v_):
        return float((oracle.pisa_attention_ex(q_, k_, v_, B, K, 1, route_eps=eps) * dO).sum())

    rng = np.random.default_rng(7)
    checked = 0
    for name, x, g in (("q", q, gq), ("k", k, gk), ("v", v, gv)):
        for _ in range(20):
            idx = (0, int(rng.integers(L)), int(rng.integers(d)))
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            if not (np.array_equal(rmask(*args_p), mask0) and np.array_equal(rmask(*args_m), mask0)):
                continue
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) <= 2e-5 * max(1.0, abs(g[idx])), (name, idx, fd, g[idx])
            checked += 1
    assert checked >= 40


@pytest.mark.parametrize("order,gate", [(0, True), (1, True), (2, True), (2, False)])
def test_backward_identities(order, gate):
    # Two exact identities of the method (PISA paper section 3.2 with the
    # blog's Taylor terms): adding one vector to every key shifts each row's
    # logits x_n, the centroid score and l_tj by the same amount (u_n and w
    # do not change), so o is unchanged and sum_n dk_n = 0; and each row's
    # weights sum to D (sum_n u_n = 0 within a block), so sum_n dv_n = sum_t dO_t.
    q, k, v = small(91 + order, BH=2, L=256, d=16, scale=3.0)
    dO = small(97, BH=2, L=256, d=16)[0]
    _, gk, gv = oracle.pisa_backward(q, k, v, dO, 32, 3, order, gate)
    scale = np.abs(gk).sum(axis=1)
    assert np.all(np.abs(gk.sum(axis=1)) <= 1e-12 * scale + 1e-13)
    np.testing.assert_allclose(gv.sum(axis=1), dO.astype(np.float64).sum(axis=1), rtol=0, atol=1e-11)


def test_backward_dq_rows_are_the_full_backward_rows():
    q, k, v = small(101, BH=2, L=256, d=16, scale=2.0)
    dO = small(103, BH=2, L=256, d=16)[0]
    for order, reps in ((1, None), (2, None), (1, 1e-6)):
        gq, _, _ = oracle.pisa_backward(q, k, v, dO, 32, 2, order, True, route_eps=reps)
        rows = [(0, 0), (0, 31), (1, 32), (1, 200), (0, 255)]
        got = oracle.pisa_backward_dq_rows(q, k, v, dO, 32, 2, rows, order, True, route_eps=reps)
        np.testing.assert_array_equal(got, np.stack([gq[b, t] for b, t in rows]))


def test_backward_with_a_given_forward_output():
    # delta_t = dO_t . o_t is the only place the forward output enters the gradient.
    # (1) given the method's own output, the gradients are those of the recomputed one
    # (up to o's rounding to fp32); (2) dv does not depend on o; (3) at K = all (dense
    # softmax attention) a change e_t of delta_t moves dq_t by -e_t sum_n P_tn k_n and dk_n
    # by -sum_t e_t P_tn q_t, P the dense softmax weights (written out here in numpy).
    L, d, B = 64, 8, 16
    q, k, v = small(111, BH=2, L=L, d=d, scale=1.5)
    dO = small(112, BH=2, L=L, d=d)[0]
    for order, gate, K in ((1, True, 1), (2, False, 2), (0, True, 1), (1, True, L // B)):
        o = oracle.pisa_attention_ex(q, k, v, B, K, order, gate=gate)
        g0 = oracle.pisa_backward(q, k, v, dO, B, K, order, gate)
        g1 = oracle.pisa_backward(q, k, v, dO, B, K, order, gate, o=o)
        for a, b in zip(g0, g1):
            assert oracle.rel_l2(b, a) <= 1e-6
    K = L // B
    o = oracle.pisa_attention_ex(q, k, v, B, K, 1).astype(np.float32)
    o2 = (o + 0.25 * np.random.default_rng(113).standard_normal(o.shape)).astype(np.float32)
    ga = oracle.pisa_backward(q, k, v, dO, B, K, 1, o=o)
    gb = oracle.pisa_backward(q, k, v, dO, B, K, 1, o=o2)
    q64, k64, dO64 = (x.astype(np.float64) for x in (q, k, dO))
    e = np.einsum("btc,btc->bt", dO64, o2.astype(np.float64) - o.astype(np.float64))
    x = q64 @ k64.transpose(0, 2, 1)
    P = np.exp(x - x.max(axis=-1, keepdims=True))
    P /= P.sum(axis=-1, keepdims=True)
    np.testing.assert_allclose(gb[0] - ga[0], -e[..., None] * (P @ k64), rtol=0, atol=1e-11)
    np.testing.assert_allclose(gb[1] - ga[1], -np.einsum("bt,btn,btc->bnc", e, P, q64), rtol=0, atol=1e-11)
    np.testing.assert_array_equal(gb[2], ga[2])


@pytest.mark.parametrize("gate", [True, False])
def test_pooled_w_backward_matches_central_differences(gate):
    # PWT's diagonal + pooled w (one w per query tile and block, from the tile mean of q^2
    # and the block's channel variances): its gradient reaches q and k through w as well;
    # coordinates whose perturbation changes the selection or a gate decision are skipped
    L, d, B, K = 64, 4, 16, 2
    q, k, v = _dyadic_qkv(131, L, d)
    q *= 2.0
    k *= 2.0
    dO = _dyadic_qkv(137, L, d)[0]
    gq, gk, gv = oracle.pisa_backward(q, k, v, dO, B, K, 2, gate, w_pooled=True)
    _, mask0, _ = oracle.select(q, k, B, K)
    h = 2.0 ** -10

    def kept(q_, k_):
        # which (tile, block) pooled w pass the ln B gate (numpy, from the definition)
        q64, k64 = q_[0].astype(np.float64), k_[0].astype(np.float64)
        q2 = (q64.reshape(-1, B, d) ** 2).mean(axis=1)
        kb = k64.reshape(-1, B, d)
        sig2 = ((kb - kb.mean(axis=1, keepdims=True)) ** 2).mean(axis=1)
        return 0.5 * q2 @ sig2.T <= math.log(B)

    keep0 = kept(q, k)
    if gate:
        assert 0 < keep0.sum() < keep0.size  # both branches of the gate are exercised

    def loss(q_, k_, v_):
        return float((oracle.pisa_attention_ex(q_, k_, v_, B, K, 2, gate=gate, w_pooled=True) * dO).sum())

    # the pooled term moves the gradient: without it dq and dk differ
    gq_exact = oracle.pisa_backward(q, k, v, dO, B, K, 2, gate)[0]
    assert oracle.rel_l2(gq_exact, gq) > 1e-3
    rng = np.random.default_rng(9)
    checked = 0
    for name, x, g in (("q", q, gq), ("k", k, gk), ("v", v, gv)):
        for _ in range(24):
            idx = (0, int(rng.integers(L)), int(rng.integers(d)))
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            if name != "v":
                if not (np.array_equal(oracle.select(args_p[0], args_p[1], B, K)[1], mask0) and
                        np.array_equal(oracle.select(args_m[0], args_m[1], B, K)[1], mask0)):
                    continue
                if gate and not (np.array_equal(kept(args_p[0], args_p[1]), keep0) and
                                 np.array_equal(kept(args_m[0], args_m[1]), keep0)):
                    continue
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) <= 2e-5 * max(1.0, abs(g[idx])), (name, idx, fd, g[idx])
            checked += 1
    assert checked >= 45
