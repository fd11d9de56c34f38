"""Seeded synthetic inputs for piecewise sparse attention.

This module only draws random numbers and shapes them into q, k, v tensors; it
holds none of the attention method's arithmetic.  Both the CPU oracle (through
the tests and the bench) and the CUDA path read the arrays it returns, so the
two sides always see bit-identical inputs.

Layout of every tensor: ``[BH, L, d]`` float32, C-contiguous, with batch and
heads folded into one leading axis (``BH = batch * heads``).  For the bf16
workloads the float32 values are rounded once to bfloat16 (round to nearest
even) and returned both as the rounded float32 values (exactly representable,
for the oracle) and as a ``torch.bfloat16`` tensor (for the GPU).

The workloads stand in for the DiT attention inputs the pages measure on
(PISA paper, section 4.1 "Models": Wan2.1, HunyuanVideo, FLUX.1), whose
activations are not available here:

* ``clustered``: block-structured keys around random centres, queries near a
  random centre (unit-test style inputs).
* ``field3d``: keys/queries from a smooth random field over a (t, h, w) video
  latent grid plus white noise (Wan- and Hunyuan-shaped).
* ``image_text``: a smooth 2D field for image tokens followed by i.i.d. text
  tokens (FLUX-shaped).

Queries are always returned pre-scaled by 1/sqrt(d): the pages fold the
softmax scale into q ("Sparse Linear Attention" blog, notation paragraph; PISA
paper section 3.1, Eq. 1 is written without a scale).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

SEED_BASE = 20260000


@dataclasses.dataclass(frozen=True)
class Workload:
    """One named input configuration."""

    name: str
    heads: int
    L: int
    d: int
    B: int
    K: int
    order: int
    dtype: str  # "f32" or "bf16"
    kind: str  # "clustered" | "field3d" | "image_text"
    seed: int
    grid: tuple = ()  # (t, h, w) for field3d, (h, w) for image_text
    n_centres: int = 0
    text_tokens: int = 0
    batch: int = 1

    @property
    def BH(self) -> int:
        return self.batch * self.heads

    @property
    def nblk(self) -> int:
        return self.L // self.B

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def k_for_sparsity(nblk: int, sparsity: float) -> int:
    """Number of exactly-computed blocks for a sparsity level.

    Sparsity is the share of blocks handled by the approximation (PISA paper,
    section 4.1 "Implementation Details"), so K = round((1 - s) * nblk).
    """
    return int(round((1.0 - sparsity) * nblk))


def workloads() -> dict:
    """The named workloads (sizes of the pages' DiT settings)."""
    w = {}
    w["c1"] = Workload("c1", heads=1, L=1024, d=64, B=64, K=4, order=1, dtype="f32",
                       kind="clustered", seed=SEED_BASE + 1, n_centres=16)
    w["c2"] = Workload("c2", heads=12, L=8192, d=64, B=64, K=16, order=1, dtype="bf16",
                       kind="clustered", seed=SEED_BASE + 2, n_centres=128)
    w["c2o2"] = w["c2"].with_(name="c2o2", order=2)
    w["c3"] = Workload("c3", heads=40, L=32768, d=128, B=64, K=77, order=1, dtype="bf16",
                       kind="field3d", seed=SEED_BASE + 3, grid=(8, 64, 64))
    w["c4"] = Workload("c4", heads=24, L=118784, d=128, B=128, K=93, order=1, dtype="bf16",
                       kind="field3d", seed=SEED_BASE + 4, grid=(29, 64, 64))
    for L, img in ((4608, (64, 64)), (16896, (128, 128))):
        nblk = L // 64
        for s in (50, 75, 90, 95):
            name = f"c5_L{L}_s{s}"
            w[name] = Workload(name, heads=24, L=L, d=128, B=64,
                               K=k_for_sparsity(nblk, s / 100.0), order=1, dtype="bf16",
                               kind="image_text", seed=SEED_BASE + 5, grid=img,
                               text_tokens=512)
    return w


def _rngs(seed: int, n: int):
    ss = np.random.SeedSequence(seed)
    return [np.random.default_rng(s) for s in ss.spawn(n)]


def _normal(rng, shape):
    return rng.standard_normal(shape, dtype=np.float32)


def _smooth_field(rng, heads: int, grid: tuple, d: int, sigma: tuple) -> np.ndarray:
    """White noise on a periodic grid, blurred by a separable Gaussian of the
    given per-axis sigma (in tokens) through the FFT, then normalised to zero
    mean and unit variance per (head, channel).  Returns [heads, prod(grid), d]."""
    ntok = int(np.prod(grid))
    out = np.empty((heads, ntok, d), dtype=np.float32)
    axes = tuple(range(1, 1 + len(grid)))
    # transfer function of the periodic Gaussian blur
    tf = np.ones([1] + [g for g in grid[:-1]] + [grid[-1] // 2 + 1], dtype=np.float32)
    for ax, (g, s) in enumerate(zip(grid, sigma)):
        f = np.fft.rfftfreq(g) if ax == len(grid) - 1 else np.fft.fftfreq(g)
        h = np.exp(-2.0 * (math.pi * f * s) ** 2).astype(np.float32)
        shape = [1] * (len(grid) + 1)
        shape[ax + 1] = h.shape[0]
        tf = tf * h.reshape(shape)
    for hh in range(heads):
        noise = _normal(rng, (d,) + tuple(grid))
        f = np.fft.rfftn(noise, axes=axes)
        f *= tf
        fld = np.fft.irfftn(f, s=grid, axes=axes).astype(np.float32)
        fld = fld.reshape(d, ntok)
        fld -= fld.mean(axis=1, keepdims=True)
        fld /= fld.std(axis=1, keepdims=True) + np.float32(1e-12)
        out[hh] = fld.T
    return out


def _clustered(w: Workload):
    r_c, r_kn, r_qc, r_qn, r_v = _rngs(w.seed, 5)
    BH, L, d = w.BH, w.L, w.d
    centres = _normal(r_c, (BH, w.n_centres, d))
    blk = (np.arange(L) // w.B) % w.n_centres
    k = centres[:, blk, :] + np.float32(0.5) * _normal(r_kn, (BH, L, d))
    pick = r_qc.integers(0, w.n_centres, size=(BH, L))
    q = np.take_along_axis(centres, pick[:, :, None], axis=1) + np.float32(0.5) * _normal(r_qn, (BH, L, d))
    v = _normal(r_v, (BH, L, d))
    return q, k, v


def _field3d(w: Workload):
    r_k, r_kn, r_q, r_qn, r_v = _rngs(w.seed, 5)
    BH, L, d = w.BH, w.L, w.d
    assert int(np.prod(w.grid)) == L
    sig = (1.0, 4.0, 4.0)
    k = _smooth_field(r_k, BH, w.grid, d, sig) + np.float32(0.3) * _normal(r_kn, (BH, L, d))
    q = _smooth_field(r_q, BH, w.grid, d, sig) + np.float32(0.3) * _normal(r_qn, (BH, L, d))
    v = _normal(r_v, (BH, L, d))
    return q, k, v


def _image_text(w: Workload):
    r_k, r_kn, r_q, r_qn, r_v, r_t = _rngs(w.seed, 6)
    BH, L, d = w.BH, w.L, w.d
    nimg = int(np.prod(w.grid))
    assert nimg + w.text_tokens == L
    sig = (4.0, 4.0)
    k = np.empty((BH, L, d), np.float32)
    q = np.empty((BH, L, d), np.float32)
    k[:, :nimg] = _smooth_field(r_k, BH, w.grid, d, sig) + np.float32(0.3) * _normal(r_kn, (BH, nimg, d))
    q[:, :nimg] = _smooth_field(r_q, BH, w.grid, d, sig) + np.float32(0.3) * _normal(r_qn, (BH, nimg, d))
    k[:, nimg:] = _normal(r_t, (BH, w.text_tokens, d))
    q[:, nimg:] = _normal(r_t, (BH, w.text_tokens, d))
    v = _normal(r_v, (BH, L, d))
    return q, k, v


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 (ties to even), returned as float32 values."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float32).numpy()


def generate(w: Workload, heads: Optional[int] = None):
    """Return (q, k, v) float32 arrays [BH, L, d]; q already divided by sqrt(d).

    For bf16 workloads the values are already rounded to bfloat16.  ``heads``
    optionally generates only the first heads (same values as the full draw
    for the clustered kind only when heads == w.heads)."""
    if heads is not None:
        w = w.with_(heads=heads)
    if w.kind == "clustered":
        q, k, v = _clustered(w)
    elif w.kind == "field3d":
        q, k, v = _field3d(w)
    elif w.kind == "image_text":
        q, k, v = _image_text(w)
    else:
        raise ValueError(w.kind)
    q *= np.float32(1.0 / math.sqrt(w.d))
    if w.dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    return (np.ascontiguousarray(q, dtype=np.float32),
            np.ascontiguousarray(k, dtype=np.float32),
            np.ascontiguousarray(v, dtype=np.float32))


def random_qkv(seed: int, BH: int, L: int, d: int, scale: float = 1.0, dtype: str = "f32"):
    """Plain i.i.d. Gaussian q, k, v (q scaled by scale/sqrt(d)) for small tests."""
    r_q, r_k, r_v = _rngs(seed, 3)
    q = _normal(r_q, (BH, L, d)) * np.float32(scale / math.sqrt(d))
    k = _normal(r_k, (BH, L, d))
    v = _normal(r_v, (BH, L, d))
    if dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    return q, k, v
