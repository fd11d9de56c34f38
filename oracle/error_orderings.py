"""Accuracy orderings of the method on the synthetic workloads (oracle only).

The PISA paper's Fig. 7 (section 4, ablation) orders the normalized L1 error
against dense attention: a block-sparse attention that drops the unselected
blocks is worst, the zeroth-order compensation is better, and the first-order
terms better still.  The PWT section of the "Sparse Linear Attention" blog
reports the gated second-order mass term lowering the error further.  The
pages measure this on model activations, which are not available here; this
script reports the same comparison on the seeded synthetic stand-ins, for
sampled query tiles.  It is a report, not a test: the orderings are
expectations about typical inputs, not identities.

    python -m oracle.error_orderings            # all workloads, a few minutes on 8 cores

Test infrastructure: it imports only the oracle, the input generators and numpy.
"""
from __future__ import annotations

import numpy as np

import oracle
import pisa_synth


def _sample_tiles(nblk: int, heads: int, per_head: int):
    idx = np.unique(np.linspace(0, nblk - 1, min(nblk, per_head)).round().astype(int))
    return [(h, int(i)) for h in range(heads) for i in idx]


def _dense_rows(q, k, v, rows):
    """Dense softmax attention for the listed (bh, t) rows, fp64 (PISA paper Eq. 1, scale in q)."""
    out = np.empty((len(rows), q.shape[2]))
    for r, (b, t) in enumerate(rows):
        x = k[b].astype(np.float64) @ q[b, t].astype(np.float64)
        e = np.exp(x - x.max())
        out[r] = (e @ v[b].astype(np.float64)) / e.sum()
    return out


def _sparse_only_rows(q, k, v, mask, B, rows):
    """Block-sparse attention that drops the unselected blocks: softmax over the
    selected blocks' keys only (the 'sparse' bar of Fig. 7)."""
    out = np.empty((len(rows), q.shape[2]))
    for r, (b, t) in enumerate(rows):
        i = t // B
        words = mask[b, i]
        nblk = k.shape[1] // B
        sel = [j for j in range(nblk) if (int(words[j // 32]) >> (j % 32)) & 1]
        if not sel:
            out[r] = np.nan
            continue
        keys = np.concatenate([np.arange(j * B, (j + 1) * B) for j in sel])
        x = k[b, keys].astype(np.float64) @ q[b, t].astype(np.float64)
        e = np.exp(x - x.max())
        out[r] = (e @ v[b, keys].astype(np.float64)) / e.sum()
    return out


def _errors(got, ref):
    d = np.abs(got - ref)
    return float(d.sum() / np.abs(ref).sum()), float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def report(name: str, heads: int, tiles_per_head: int, orders=(0, 1, 2)):
    w = pisa_synth.workloads()[name].with_(heads=heads)
    q, k, v = pisa_synth.generate(w)
    B, Kb = w.B, w.K
    tiles = _sample_tiles(w.nblk, heads, tiles_per_head)
    rows = [(b, i * B + m) for b, i in tiles for m in range(B)]
    ref = _dense_rows(q, k, v, rows)
    _, mask, _ = oracle.select(q, k, B, Kb)
    res = {"sparse only": _errors(_sparse_only_rows(q, k, v, mask, B, rows), ref)}
    for o in orders:
        got = oracle.pisa_attention_ex(q, k, v, B, Kb, o, gate=True, tiles=tiles).reshape(len(rows), -1)
        res[f"order {o}" + (" (gated w)" if o == 2 else "")] = _errors(got, ref)
    got = oracle.pisa_attention_ex(q, k, v, B, Kb, 1, hybrid=True, tiles=tiles).reshape(len(rows), -1)
    res["hybrid (global H-bar)"] = _errors(got, ref)
    got = oracle.pisa_attention_ex(q, k, v, B, Kb, 1, route_eps=1e-6, tiles=tiles).reshape(len(rows), -1)
    res["order 1, covariance-aware routing"] = _errors(got, ref)
    return w, len(tiles), res


def main():
    # (workload, heads, sampled query tiles per head)
    cases = [("c1", 1, 16), ("c2", 2, 16), ("c3", 1, 12), ("c5_L4608_s90", 2, 24), ("c5_L4608_s50", 2, 24),
             ("c4", 1, 8)]
    print("| workload | sampled tiles | variant | normalized L1 error | rel-L2 error |")
    print("|---|---|---|---|---|")
    for name, heads, per_head in cases:
        w, nt, res = report(name, heads, per_head)
        label = f"{name} (L={w.L}, d={w.d}, B={w.B}, K={w.K} of {w.nblk}, {w.dtype})"
        for variant, (l1, l2) in res.items():
            print(f"| {label} | {nt} | {variant} | {l1:.4f} | {l2:.4f} |")
            label = ""


if __name__ == "__main__":
    main()
