"""Host logic of bench.py (CPU only): the FLOP and byte counts its roofline figures
rest on, checked against direct counts on small selections."""
import numpy as np
import torch

import bench
import oracle
import pisa_synth


def _mask_and_union(w, seed):
    q, k, _ = pisa_synth.random_qkv(seed, w.BH, w.L, w.d, scale=2.0)
    _, mask, _ = oracle.select(q, k, w.B, w.K)
    nqt = 256 // w.B
    unions = []
    for bh in range(w.BH):
        for c0 in range(0, (w.L + 255) // 256 * nqt, nqt):
            tiles = [min(t, w.nblk - 1) for t in range(c0, c0 + nqt)]
            sel = set()
            for t in tiles:
                for j in range(w.nblk):
                    if (mask[bh, t, j // 32] >> (j % 32)) & 1:
                        sel.add(j)
            unions.append(len(sel))
    return torch.from_numpy(mask.view(np.int32)), np.array(unions)


def test_unions_and_executed_flops_match_a_direct_count():
    for d, B, L, K in [(64, 64, 2048, 5), (128, 128, 1152, 2), (128, 64, 1152, 3)]:
        w = pisa_synth.workloads()["c2"].with_(heads=2, L=L, d=d, B=B, K=K)
        mask, unions = _mask_and_union(w, 7 + d + B)
        assert np.array_equal(bench.cta_unions(w, mask).ravel(), unions)
        bpt, gb = 128 // B, (2 if d == 64 else 1)
        stc = sum(256 * (4 * d * 128 * -(-u // bpt) + 2 * d * (gb * d + 16) * -(-(w.nblk - u) // gb))
                  for u in unions)
        assert bench.stc_executed_flops(w, mask) == stc
        hyb = sum(256 * (4 * d * 128 * (-(-u // bpt) + -(-w.nblk // 128)) + 2 * d * d) for u in unions)
        assert bench.hybrid_executed_flops(w, mask) == hyb


def test_algorithmic_flops_of_the_wan_shape():
    # exact 4 L K B d + centroid scores 2 L nblk d + zeroth 2 L nU d + first 2 L nU d^2, 40 heads:
    # 22.31 TFLOP at the Wan shape (order 1)
    w = pisa_synth.workloads()["c3"]
    assert abs(bench.algorithmic_flops(w) / 1e12 - 22.31) < 0.01
    w2 = pisa_synth.workloads()["c2o2"]
    nU = w2.nblk - w2.K
    assert bench.algorithmic_flops(w2) - bench.algorithmic_flops(w2.with_(order=1)) == \
        2.0 * w2.L * nU * w2.d * w2.d * w2.BH
