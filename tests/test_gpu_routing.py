"""GPU parity of the covariance-aware routing (PISA paper, section 3.3
"Covariance-Aware Block Selection"; "Sparse Linear Attention" blog, PWT
section): the routing bias ln(||H_j||_F + eps) and the biased selection are
bit-exact against the CPU oracle; the attention with routing on is within the
path's tolerance of the oracle on every path, pooled, per row and per element
(tests/parity.py).
"""
import numpy as np
import pytest
import torch

import block_sparse_taylor_b200 as pisa
import oracle
import parity
import pisa_synth

pytestmark = pytest.mark.gpu

TDT = {"f32": torch.float32, "bf16": torch.bfloat16}
TOL = {"f32": 1e-4, "bf16": 2e-2}


def dev(x, dt):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(TDT[dt])


def gpu_bias(k, v, B, dt, eps=pisa.ROUTE_EPS):
    kt, vt = dev(k, dt), dev(v, dt)
    st = pisa.pisa_centroids(kt, B)
    bias = pisa.pisa_route_bias(kt, vt, st.kbar, B, eps)
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    return st, bias


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (64, 128), (128, 128)])
def test_route_bias_bit_exact(dt, d, B):
    q, k, v = pisa_synth.random_qkv(700 + d + B, 2, 1024, d, scale=1.0, dtype=dt)
    _, bias = gpu_bias(k, v, B, dt)
    np.testing.assert_array_equal(bias.cpu().numpy(), oracle.route_bias(k, v, B))


@pytest.mark.parametrize("eps", [1e-6, 0.25, 40.0])
def test_route_bias_eps_and_constant_blocks(eps):
    # blocks of identical keys have H_j = 0: their bias is ln(eps) exactly as the oracle computes it
    rng = np.random.default_rng(11)
    B, d, nblk = 64, 64, 8
    k = np.repeat(rng.standard_normal((1, nblk, 1, d)), B, axis=2).reshape(1, nblk * B, d).astype(np.float32)
    k[:, 2 * B:3 * B] += rng.standard_normal((1, B, d)).astype(np.float32)  # one heterogeneous block
    v = rng.standard_normal((1, nblk * B, d)).astype(np.float32)
    _, bias = gpu_bias(k, v, B, "f32", eps)
    want = oracle.route_bias(k, v, B, eps)
    np.testing.assert_array_equal(bias.cpu().numpy(), want)
    lneps = oracle.ln_f32(np.array([eps], np.float32))[0]
    assert np.all(want[0, [0, 1, 3, 4, 5, 6, 7]] == lneps) and want[0, 2] > lneps


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d,B,L", [(64, 64, 2048), (128, 64, 4096), (128, 128, 4096), (64, 64, 576)])
@pytest.mark.parametrize("Kfrac", [0.1, 0.5])
def test_biased_selection_bit_exact(dt, d, B, L, Kfrac):
    q, k, v = pisa_synth.random_qkv(800 + d + B + L, 2, L, d, scale=1.0, dtype=dt)
    nblk = L // B
    K = max(1, int(round(Kfrac * nblk)))
    st, bias = gpu_bias(k, v, B, dt)
    idx, mask = pisa.pisa_select(dev(q, dt), st, K, bias=bias)
    torch.cuda.synchronize()
    ridx, rmask, _ = oracle.select(q, k, B, K, bias=oracle.route_bias(k, v, B))
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(mask.cpu().numpy().view(np.uint32), rmask)
    if L >= 2048:
        # routing changes the selection on these inputs (the test would be vacuous otherwise)
        pidx, _, _ = oracle.select(q, k, B, K)
        assert not np.array_equal(pidx, ridx)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d,B", [(64, 64), (128, 128)])
def test_biased_scores_bit_exact(dt, d, B):
    q, k, v = pisa_synth.random_qkv(850 + d + B, 2, 2048, d, scale=1.0, dtype=dt)
    st, bias = gpu_bias(k, v, B, dt)
    sc = pisa.pisa_select_scores(dev(q, dt), st, bias)
    torch.cuda.synchronize()
    _, _, ref = oracle.select(q, k, B, 1, want_scores=True, bias=oracle.route_bias(k, v, B))
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("name,heads", [("c3", 2), ("c4", 1), ("c2", 3)])
def test_routing_full_size_bit_exact(name, heads):
    w = pisa_synth.workloads()[name].with_(heads=heads)
    q, k, v = pisa_synth.generate(w)
    st, bias = gpu_bias(k, v, w.B, w.dtype)
    rbias = oracle.route_bias(k, v, w.B)
    np.testing.assert_array_equal(bias.cpu().numpy(), rbias)
    idx, mask = pisa.pisa_select(dev(q, w.dtype), st, w.K, bias=bias)
    torch.cuda.synchronize()
    ridx, rmask, _ = oracle.select(q, k, w.B, w.K, bias=rbias)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(mask.cpu().numpy().view(np.uint32), rmask)


@pytest.mark.parametrize("path,dt", [("recompute_tc", "bf16"), ("stats", "bf16"), ("stats", "f32"),
                                     ("hybrid_tc", "bf16"), ("stats_tc", "bf16")])
@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (128, 128)])
def test_attention_with_routing(path, dt, d, B):
    L = 1024
    q, k, v = pisa_synth.random_qkv(900 + d + B, 2, L, d, scale=2.0, dtype=dt)
    K = (L // B) // 4
    out = pisa.pisa_attention(dev(q, dt), dev(k, dt), dev(v, dt), B, K, 1, path=path, route="cov")
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    got = out.float().cpu().numpy()
    ref = oracle.pisa_attention_ex(q, k, v, B, K, 1, hybrid=(path == "hybrid_tc"), route_eps=pisa.ROUTE_EPS)
    parity.check(got, ref, dt, path)
    # routing changed the oracle's result here (the comparison would be vacuous otherwise)
    plain = oracle.pisa_attention_ex(q, k, v, B, K, 1, hybrid=(path == "hybrid_tc"))
    assert oracle.rel_l2(plain, ref) > 1e-6
