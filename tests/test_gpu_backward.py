"""GPU parity of the backward pass (pisa_attention_backward) against the CPU
oracle's gradients.

The pages define only the forward (PISA paper section 3.2 "Formulation";
"Sparse Linear Attention" blog, sparse-linear and PWT sections); both sides
differentiate it with the block selection held fixed (and, for order 2, the
gate decision).  The oracle's gradients are pinned in test_oracle_pins.py
(central differences, autograd of dense attention at K = all, exact identities).

The backward is an operator of (q, k, v, o, dO): the forward output o enters
only through delta_t = dO_t . o_t.  The oracle is given the same o the GPU
received (in the input dtype), so each comparison measures the backward's own
arithmetic; test_backward_parity also compares with the oracle's exact-o
gradients under the pooled bound (bf16 o moves delta by up to 2^-9 |dO_t||o_t|,
and at order 2 the u_n / B term of dS amplifies that in a few rows to a few
per cent, which a rounding model of the kernel with otherwise exact arithmetic
reproduces).

Tolerances (rel-L2 per gradient tensor, and the per-row and per-element bounds
of tests/parity.py): fp32 inputs 1e-4 (fp32 arithmetic throughout, fp32
accumulation over L keys); bf16 inputs 2e-2 (P and dS are rounded to bf16 as
operands of the dk, dv and dq products).
"""
import math

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


def inputs(seed, BH, L, d, dt, scale=2.0):
    q, k, v = pisa_synth.random_qkv(seed, BH, L, d, scale=scale, dtype=dt)
    dO = pisa_synth.random_qkv(seed + 1, BH, L, d, scale=1.0, dtype=dt)[0]
    return q, k, v, dO


def gpu_backward(q, k, v, od, dO, B, K, order, gate, dt, route="centroid"):
    """The library's gradients; ``od`` is the forward output on the device (input dtype)."""
    grads = pisa.pisa_attention_backward(dev(q, dt), dev(k, dt), dev(v, dt), od, dev(dO, dt), B, K, order,
                                         gate=gate, route=route)
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    return [g.cpu().numpy().astype(np.float64) for g in grads]


def host(od):
    """A device forward output as the fp32 numpy array the oracle takes."""
    return od.detach().float().cpu().numpy()


def check(got, want, dt):
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        parity.check(g, w, dt, name, grad=True)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("order,gate", [(0, True), (1, True), (2, True), (2, False)])
def test_backward_parity(dt, d, B, order, gate):
    L = 1024
    q, k, v, dO = inputs(1100 + d + B + 10 * order, 2, L, d, dt, scale=3.0 if order == 2 else 2.0)
    K = (L // B) // 4
    od = dev(oracle.pisa_attention_ex(q, k, v, B, K, order, gate=gate), dt)
    got = gpu_backward(q, k, v, od, dO, B, K, order, gate, dt)
    check(got, oracle.pisa_backward(q, k, v, dO, B, K, order, gate, o=host(od)), dt)
    # against the exact gradient (delta from the fp64 o): the pooled bound
    for g, w in zip(got, oracle.pisa_backward(q, k, v, dO, B, K, order, gate)):
        assert oracle.rel_l2(g, w) <= TOL[dt]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("L,B", [(576, 64), (640, 128), (64, 64), (128, 128)])
def test_backward_ragged_and_tiny_lengths(dt, L, B):
    # lengths that are not a multiple of the 128-row forward tile, and a single block
    d = 64
    q, k, v, dO = inputs(1200 + L + B, 2, L, d, dt)
    K = max(1, (L // B) // 3)
    od = dev(oracle.pisa_attention_ex(q, k, v, B, K, 1), dt)
    got = gpu_backward(q, k, v, od, dO, B, K, 1, True, dt)
    check(got, oracle.pisa_backward(q, k, v, dO, B, K, 1, o=host(od)), dt)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("K", ["none", "all"])
@pytest.mark.parametrize("order", [1, 2])
def test_backward_degenerate_selections(dt, K, order):
    # K = 0: every block through its Taylor term; K = all: exact dense attention
    L, d, B = 512, 64, 64
    Kv = 0 if K == "none" else L // B
    q, k, v, dO = inputs(1300 + order + Kv, 2, L, d, dt)
    od = dev(oracle.pisa_attention_ex(q, k, v, B, Kv, order), dt)
    got = gpu_backward(q, k, v, od, dO, B, Kv, order, True, dt)
    check(got, oracle.pisa_backward(q, k, v, dO, B, Kv, order, o=host(od)), dt)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d,B", [(64, 64), (128, 128)])
def test_backward_with_routing(dt, d, B):
    # covariance-aware selection recomputed inside the backward (bit-exact routing
    # and selection), gradients on that selection
    L = 1024
    q, k, v, dO = inputs(1400 + d + B, 2, L, d, dt)
    K = (L // B) // 4
    od = dev(oracle.pisa_attention_ex(q, k, v, B, K, 1, route_eps=pisa.ROUTE_EPS), dt)
    got = gpu_backward(q, k, v, od, dO, B, K, 1, True, dt, route="cov")
    want = oracle.pisa_backward(q, k, v, dO, B, K, 1, True, route_eps=pisa.ROUTE_EPS, o=host(od))
    check(got, want, dt)
    plain = oracle.pisa_backward(q, k, v, dO, B, K, 1)
    assert oracle.rel_l2(plain[0], want[0]) > 1e-3  # routing reaches the gradient on these inputs


@pytest.mark.parametrize("path", ["recompute_tc", "stats"])
def test_forward_then_backward_on_the_gpu(path):
    # the training use: o from the library's own forward, then the backward
    dt, L, d, B, order = "bf16", 1024, 128, 64, 1
    q, k, v, dO = inputs(1500, 2, L, d, dt)
    K = (L // B) // 4
    o = pisa.pisa_attention(dev(q, dt), dev(k, dt), dev(v, dt), B, K, order, path=path)
    grads = pisa.pisa_attention_backward(dev(q, dt), dev(k, dt), dev(v, dt), o, dev(dO, dt), B, K, order)
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    check([g.cpu().numpy().astype(np.float64) for g in grads],
          oracle.pisa_backward(q, k, v, dO, B, K, order, o=host(o)), dt)


def test_backward_overwrites_its_outputs_and_repeats_bit_for_bit():
    dt, L, d, B = "bf16", 512, 64, 64
    q, k, v, dO = inputs(1600, 2, L, d, dt)
    o = oracle.pisa_attention_ex(q, k, v, B, 2, 1)
    args = [dev(x, dt) for x in (q, k, v, o, dO)]
    first = [g.clone() for g in pisa.pisa_attention_backward(*args, B, 2)]
    grads = tuple(torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda") for _ in range(3))
    again = pisa.pisa_attention_backward(*args, B, 2, grads=grads)
    torch.cuda.synchronize()
    for a, b in zip(first, again):
        assert torch.equal(a, b)


@pytest.mark.parametrize("name,heads", [("c3", 1), ("c2", 1)])
def test_backward_full_size_sampled_rows_and_identities(name, heads):
    # Full sequence length and block size of the workload, in the launch
    # configuration bench.py times.  The oracle computes sampled dq rows one by
    # one; dk and dv are checked through two exact identities of the method:
    # sum_n dk_n = 0 (a common shift of all keys leaves o unchanged) and
    # sum_n dv_n = sum_t dO_t (each row's weights sum to D).
    w = pisa_synth.workloads()[name].with_(heads=heads)
    q, k, v = pisa_synth.generate(w)
    dt = w.dtype
    BH, L, d = q.shape
    dO = pisa_synth.random_qkv(1700, BH, L, d, scale=1.0, dtype=dt)[0]
    qd, kd, vd, dOd = dev(q, dt), dev(k, dt), dev(v, dt), dev(dO, dt)
    o = pisa.pisa_attention(qd, kd, vd, w.B, w.K, w.order)
    dq, dk, dv = pisa.pisa_attention_backward(qd, kd, vd, o, dOd, w.B, w.K, w.order)
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    rng = np.random.default_rng(17)
    rows = [(int(rng.integers(BH)), int(t)) for t in rng.integers(0, L, 24)] + [(0, 0), (BH - 1, L - 1)]
    want = oracle.pisa_backward_dq_rows(q, k, v, dO, w.B, w.K, rows, w.order, o=host(o))
    got = np.stack([dq[b, t].cpu().numpy().astype(np.float64) for b, t in rows])
    parity.check(got, want, dt, "dq rows", grad=True)
    dk64, dv64 = dk.double(), dv.double()
    for b in range(BH):
        assert float(dk64[b].sum(0).norm()) <= 1e-2 * float(dk64[b].norm(dim=1).sum())
        s_dv, s_do = dv64[b].sum(0), dOd[b].double().sum(0)
        assert float((s_dv - s_do).norm()) <= 1e-2 * float(s_do.norm()) + 1e-3 * math.sqrt(L)


def test_autograd_function():
    # pisa_attention_autograd: gradients through torch.autograd equal the entry point's (cast to
    # the input dtype) and match the oracle
    dt, L, d, B, K = "bf16", 1024, 128, 64, 4
    q, k, v, dO = inputs(1800, 2, L, d, dt)
    qt, kt, vt = (dev(x, dt).requires_grad_() for x in (q, k, v))
    out = pisa.pisa_attention_autograd(qt, kt, vt, B, K, 1)
    out.backward(dev(dO, dt))
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    # the autograd function hands the backward its forward's lse; the same deterministic
    # forward gives the same lse here
    _, lse = pisa.pisa_attention_lse(dev(q, dt), dev(k, dt), dev(v, dt), B, K, 1)
    direct = pisa.pisa_attention_backward(dev(q, dt), dev(k, dt), dev(v, dt), out.detach(), dev(dO, dt), B, K, 1,
                                          lse=lse)
    for t, g in zip((qt, kt, vt), direct):
        assert t.grad.dtype == torch.bfloat16
        assert torch.equal(t.grad, g.to(torch.bfloat16))
    check([t.grad.float().cpu().numpy().astype(np.float64) for t in (qt, kt, vt)],
          oracle.pisa_backward(q, k, v, dO, B, K, 1, o=host(out)), dt)
    with pytest.raises(pisa.PisaError):
        pisa.pisa_attention_autograd(qt, kt, vt, B, K, 1, path="hybrid_tc")


def test_autograd_four_dimensional_inputs_with_routing_and_order2():
    # [batch, heads, L, d] tensors through the autograd wrapper; covariance-aware routing and
    # the gated second order; compared with the oracle on the folded [batch*heads, L, d] view
    dt, L, d, B, K = "bf16", 512, 64, 64, 2
    q, k, v, dO = inputs(1850, 6, L, d, dt, scale=3.0)
    shape4 = (2, 3, L, d)
    qt, kt, vt = (dev(x, dt).reshape(shape4).requires_grad_() for x in (q, k, v))
    out = pisa.pisa_attention_autograd(qt, kt, vt, B, K, 2, route="cov")
    assert out.shape == shape4
    out.backward(dev(dO, dt).reshape(shape4))
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    want_o = oracle.pisa_attention_ex(q, k, v, B, K, 2, route_eps=pisa.ROUTE_EPS)
    parity.check(out.detach().float().reshape(6, L, d).cpu().numpy(), want_o, dt, "o")
    got = [t.grad.float().reshape(6, L, d).cpu().numpy().astype(np.float64) for t in (qt, kt, vt)]
    check(got, oracle.pisa_backward(q, k, v, dO, B, K, 2, True, route_eps=pisa.ROUTE_EPS,
                                    o=host(out).reshape(6, L, d)), dt)


@pytest.mark.parametrize("path,dt", [("recompute_tc", "bf16"), ("stats_tc", "bf16"), ("stats", "bf16"),
                                     ("stats", "f32")])
def test_forward_lse_is_the_log_denominator(path, dt):
    # pisa_attention_lse: ln D_t of the shared denominator, against the oracle's log D_t
    L, d, B, K = 1024, 64, 64, 4
    q, k, v = pisa_synth.random_qkv(1910, 2, L, d, scale=2.0, dtype=dt)
    out, lse = pisa.pisa_attention_lse(dev(q, dt), dev(k, dt), dev(v, dt), B, K, 1, path=path)
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    ref_o, ref_lse = oracle.pisa_attention(q, k, v, B, K, 1, want_lse=True)
    parity.check(out.float().cpu().numpy(), ref_o, dt, "o")
    tol = 1e-5 if dt == "f32" else 2e-3  # absolute, in natural-log units (a relative 2e-3 of D)
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= tol


@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("order", [0, 1, 2])
def test_backward_with_the_forwards_lse(d, B, order):
    # the tensor-core backward given the forward's log-denominators: no row-statistics pass
    dt, L = "bf16", 1024
    q, k, v, dO = inputs(1950 + d + B + order, 2, L, d, dt, scale=3.0 if order == 2 else 2.0)
    K = (L // B) // 4
    qd, kd, vd, dOd = dev(q, dt), dev(k, dt), dev(v, dt), dev(dO, dt)
    o, lse = pisa.pisa_attention_lse(qd, kd, vd, B, K, order)
    grads = pisa.pisa_attention_backward(qd, kd, vd, o, dOd, B, K, order, lse=lse)
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    check([g.cpu().numpy().astype(np.float64) for g in grads],
          oracle.pisa_backward(q, k, v, dO, B, K, order, o=host(o)), dt)


def _pooled_inputs(seed, d, B, L=1024):
    # half of the key blocks 1.4 times wider: their pooled w lands above ln B, the others'
    # below, so both branches of the gate run, every (tile, block) pair well clear of it
    q, k, v, dO = inputs(seed, 2, L, d, "bf16", scale=2.4)
    kk = k.reshape(2, L // B, B, d).copy()
    kk[:, 1::2] *= 1.4
    k = pisa_synth.round_bf16(kk.reshape(2, L, d))
    q64, k64 = q.astype(np.float64), k.astype(np.float64)
    q2 = (q64.reshape(2, -1, B, d) ** 2).mean(axis=2)
    kb = k64.reshape(2, -1, B, d)
    var = ((kb - kb.mean(axis=2, keepdims=True)) ** 2).mean(axis=2)
    w = 0.5 * np.einsum("bic,bjc->bij", q2, var)
    assert np.abs(w - math.log(B)).min() > 0.05 * math.log(B)
    assert 0.2 < (w > math.log(B)).mean() < 0.8
    return q, k, v, dO


@pytest.mark.parametrize("d,B", [(64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("gate", [True, False])
def test_pooled_w_backward(d, B, gate):
    # PWT's diagonal + pooled w at order 2 (the forward's pooled path, then the backward with
    # its lse): the pooled w's gradient reaches q and k through the tile means of q^2 and the
    # blocks' channel variances
    dt, L = "bf16", 1024
    q, k, v, dO = _pooled_inputs(2300 + d + B, d, B, L)
    K = (L // B) // 4
    qd, kd, vd, dOd = dev(q, dt), dev(k, dt), dev(v, dt), dev(dO, dt)
    o, lse = pisa.pisa_attention_lse(qd, kd, vd, B, K, 2, gate=gate, w_mode="pooled")
    grads = pisa.pisa_attention_backward(qd, kd, vd, o, dOd, B, K, 2, gate=gate, lse=lse, w_mode="pooled")
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    parity.check(o.float().cpu().numpy(), oracle.pisa_attention_ex(q, k, v, B, K, 2, gate=gate, w_pooled=True),
                 dt, "o")
    want = oracle.pisa_backward(q, k, v, dO, B, K, 2, gate, o=host(o), w_pooled=True)
    check([g.cpu().numpy().astype(np.float64) for g in grads], want, dt)
    # the pooled w's gradient is a visible part of dq and dk on these inputs
    plain = oracle.pisa_backward(q, k, v, dO, B, K, 1, gate, o=host(o))
    assert oracle.rel_l2(plain[0], want[0]) > 1e-2 and oracle.rel_l2(plain[1], want[1]) > 1e-2


def test_pooled_w_backward_repeats_bit_for_bit_and_through_autograd():
    dt, L, d, B, K = "bf16", 1024, 128, 64, 4
    q, k, v, dO = _pooled_inputs(2400, d, B, L)
    qt, kt, vt = (dev(x, dt).requires_grad_() for x in (q, k, v))
    out = pisa.pisa_attention_autograd(qt, kt, vt, B, K, 2, w_mode="pooled")
    out.backward(dev(dO, dt))
    _, lse = pisa.pisa_attention_lse(dev(q, dt), dev(k, dt), dev(v, dt), B, K, 2, w_mode="pooled")
    args = (dev(q, dt), dev(k, dt), dev(v, dt), out.detach(), dev(dO, dt), B, K, 2)
    first = pisa.pisa_attention_backward(*args, lse=lse, w_mode="pooled")
    again = pisa.pisa_attention_backward(*args, lse=lse, w_mode="pooled")
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()
    for t, a, b in zip((qt, kt, vt), first, again):
        assert torch.equal(a, b)  # fixed-order sums: the same result on every run
        assert torch.equal(t.grad, a.to(torch.bfloat16))
    with pytest.raises(pisa.PisaError):  # the pooled-w backward takes the forward's lse
        pisa.pisa_attention_backward(*args, w_mode="pooled")
