#!/usr/bin/env python
"""Benchmark of piecewise sparse attention on B200.

One step = one forward pass of the whole hot path on one batch of synthetic
input: block centroids -> top-K block selection -> fused attention (exact
blocks, Taylor-compensated unselected blocks, normalisation), i.e. exactly the
kernels ``pisa_attention`` runs, called stage by stage through the C ABI so
that each kernel is bracketed by CUDA events on the launching stream.

Default workload: Wan2.1-shaped attention, 1 x 40 heads, L = 32768, d = 128,
bf16, B = 64, K = 77, order 1 (inputs 1 GiB > L2, so no flush is needed
between steps).  Metric: full-attention-equivalent TFLOP/s, 4 L^2 d H / t,
whole job.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                       [--shard heads|replicas]
Multi-GPU: one rank per GPU.  Under torch.distributed.run WORLD_SIZE must equal
--gpus; without it, --gpus N > 1 starts N ranks through torch.distributed.run
itself.  --shard heads (default): the workload's (batch, head) units are split
across the ranks, each rank times its own slice with the unchanged single-GPU
call, and the value is the whole workload over the slowest rank's time (strong
scaling; no collective on the data path).  --shard replicas: every rank runs
the whole workload on its own inputs (weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/call & full-attn-equiv TFLOP/s at Wan-shape L=32K; % of roofline"
UNIT = "TFLOP/s (full-attention-equivalent, 4*L^2*d*heads per call)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="c3")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--heads", type=int, default=None, help="override head count (profiling small cases)")
    p.add_argument("--no-hybrid", action="store_true", help="skip the PISA-hybrid (global H-bar) record")
    p.add_argument("--no-route", action="store_true", help="skip the covariance-aware routing record")
    p.add_argument("--no-backward", action="store_true", help="skip the backward-pass record")
    p.add_argument("--no-dense", action="store_true", help="skip the dense-SDPA context record")
    p.add_argument("--shard", default="heads", choices=["heads", "replicas"],
                   help="multi-GPU split: the workload's heads across ranks, or one replica per rank")
    return p.parse_args()


def world_plan(gpus: int, env) -> str:
    """"run" when the process layout matches --gpus, "launch" when N > 1 ranks must be
    started (no torch.distributed.run around this process); raises SystemExit when
    WORLD_SIZE contradicts --gpus."""
    if gpus < 1:
        raise SystemExit(f"--gpus must be >= 1 (got {gpus})")
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != gpus:
            raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}: launch one rank per GPU")
        return "run"
    return "launch" if gpus > 1 else "run"


def launch_ranks(gpus: int) -> int:
    """Start --gpus ranks of this same command through torch.distributed.run (one node,
    rendezvous on 127.0.0.1) and return their exit status."""
    import socket

    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def pct(sorted_vals, p):
    """p-th percentile of an ascending list (linear interpolation)."""
    if not sorted_vals:
        return None
    x = (len(sorted_vals) - 1) * p / 100.0
    lo = int(x)
    hi = min(lo + 1, len(sorted_vals) - 1)
    return sorted_vals[lo] + (sorted_vals[hi] - sorted_vals[lo]) * (x - lo)


def dense_sdpa_record(q, k, v, stream, reps=3):
    """Context only, not a target: torch's dense scaled_dot_product_attention (a library kernel:
    flash, cuDNN or memory-efficient backend, never the L^2-memory math one) on the same inputs,
    q already scaled.  Any failure is reported, not raised."""
    try:
        import torch
        import torch.nn.functional as F
        from torch.nn.attention import SDPBackend, sdpa_kernel

        qd, kd, vd = (x.unsqueeze(0) for x in (q, k, v))
        with sdpa_kernel([SDPBackend.FLASH_ATTENTION, SDPBackend.CUDNN_ATTENTION, SDPBackend.EFFICIENT_ATTENTION]):
            F.scaled_dot_product_attention(qd, kd, vd, scale=1.0)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                F.scaled_dot_product_attention(qd, kd, vd, scale=1.0)
            b.record(stream)
            torch.cuda.synchronize()
        return {"ms_per_call": a.elapsed_time(b) / reps, "calls_timed": reps,
                "note": "torch scaled_dot_product_attention, dense, library kernel; context only"}
    except Exception as e:  # noqa: BLE001 - a context record never fails the benchmark
        return {"unavailable": f"{type(e).__name__}: {e}"[:240]}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("attn_tc.cuh", "tc_ptx.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "block_sparse_taylor_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_record(workload: str):
    """DRAM bytes per launch of the attention kernel from a committed ncu
    summary, only if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", f"attn_tc_{workload}_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("source_sha256") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        loaded = [x for x in sm if x > 0.5 * (mx or 1)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's value (timings are reported as the max over ranks)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def rank_workload(w, rank: int):
    """Weak scaling: rank r runs the same workload on its own seeded inputs
    (rank 0 keeps the canonical seed)."""
    return w.with_(seed=w.seed + 1000 * rank) if rank else w


def cpu_baseline(w, q, k, v, tiles_per_thread=4):
    """Time the CPU oracle, as it stands, on a bounded sample of the workload:
    the block statistics of head 0 plus a few query tiles of head 0 (spread
    evenly, first and last included), extrapolated to the whole call (all
    heads, all tiles).  The oracle's output rows of those tiles are returned
    under "_ref" for the parity record."""
    import oracle

    nthreads = oracle.default_threads()
    qh, kh, vh = q[:1], k[:1], v[:1]
    t0 = time.perf_counter()
    oracle.block_stats(kh, vh, w.B, order=w.order, nthreads=nthreads)
    t_stats = time.perf_counter() - t0
    ntiles = max(1, min(w.nblk, tiles_per_thread * nthreads))
    tiles = sorted({(0, int(i)) for i in np.linspace(0, w.nblk - 1, ntiles).round()})
    t0 = time.perf_counter()
    ref = oracle.pisa_attention(qh, kh, vh, w.B, w.K, w.order, tiles=tiles, nthreads=nthreads)
    t_call = time.perf_counter() - t0
    # oracle.pisa_attention also recomputes the head's statistics and selection
    t_tiles = max(t_call - t_stats, 1e-9)
    per_tile = t_tiles / len(tiles)
    # the oracle computes the statistics of different heads on different threads
    t_full = w.BH * (t_stats / min(nthreads, w.BH) + per_tile * w.nblk)
    flops = 4.0 * w.L * w.L * w.d * w.BH
    return {
        "value": flops / t_full / 1e12,
        "unit": UNIT,
        "cores": nthreads,
        "kind": "oracle",
        "sample": (f"head 0 of {w.BH}: block statistics ({t_stats:.2f} s) + {len(tiles)} of {w.nblk} query tiles "
                   f"({t_tiles:.2f} s, includes re-running that head's statistics and selection); extrapolated to "
                   f"{w.BH} heads x {w.nblk} tiles = {t_full:.0f} s per call"),
        "seconds_measured": t_stats + t_call,
        "_ref": (tiles, ref),
    }


def parity_record(w, out, mask, q_h, k_h, ref_tiles):
    """The timed step's output against the oracle on the sampled tiles of head 0 (rel-L2, worst
    row, worst element; tolerance 2e-2 bf16 / 1e-4 fp32), and the GPU selection of head 0
    against the oracle's canonical selection (every query tile; must be 0 mismatches)."""
    import oracle

    tiles, ref = ref_tiles
    B = w.B
    got = np.stack([out[bh, i * B:(i + 1) * B].float().cpu().numpy() for bh, i in tiles])
    m = oracle.parity_metrics(got, ref)
    _, rmask, _ = oracle.select(q_h[:1], k_h[:1], B, w.K)
    gmask = mask[0].cpu().numpy().view(np.uint32)
    bad_tiles = int(np.sum(np.any(gmask != rmask[0], axis=1)))
    bad_bits = int(sum(bin(int(x)).count("1") for x in np.bitwise_xor(gmask, rmask[0]).ravel()))
    tol = 2e-2 if w.dtype == "bf16" else 1e-4
    return {"rows_compared": m["rows"], "tiles": f"{len(tiles)} query tiles of head 0 (first, last, evenly spread)",
            "rel_l2": m["rel_l2"], "row_max": m["row_max"], "elem_max": m["elem_max"], "tolerance": tol,
            "within_tolerance": bool(m["rel_l2"] <= tol and m["row_max"] <= tol and m["elem_max"] <= tol),
            "selection_mismatches": bad_tiles, "selection_bits_differing": bad_bits,
            "selection_tiles_compared": int(gmask.shape[0])}


def cpu_backward_baseline(w, q, k, v, dO):
    """Time the oracle's backward, as it stands, on a bounded sample: dq of sampled query rows of
    head 0, one row per thread, in calls of n and 8n rows so that the head's selection and
    centroids (computed once per call) separate from the per-row cost.  Extrapolated the way the
    oracle's whole backward runs (heads in parallel, each head's rows in series).  That backward
    also accumulates dk and dv for every row, so the estimate is a lower bound on its time."""
    import oracle

    nt = oracle.default_threads()
    qh, kh, vh, dh = q[:1], k[:1], v[:1], dO[:1]

    def timed(n):
        rows = [(0, int(t)) for t in np.linspace(0, w.L - 1, n).round()]
        t0 = time.perf_counter()
        oracle.pisa_backward_dq_rows(qh, kh, vh, dh, w.B, w.K, rows, w.order, nthreads=nt)
        return time.perf_counter() - t0

    t1, t8 = timed(nt), timed(8 * nt)
    c_row = max((t8 - t1) / 7.0, 1e-9)
    prep = max(t1 - c_row, 0.0)
    t_full = math.ceil(w.BH / nt) * (prep + w.L * c_row)
    flops = 10.0 * w.L * w.L * w.d * w.BH
    return {"value": flops / t_full / 1e12, "unit": "TFLOP/s (algorithmic backward, 10*L^2*d*heads per call)",
            "cores": nt, "kind": "oracle",
            "sample": (f"head 0 of {w.BH}: dq of {nt} and {8 * nt} sampled rows ({t1:.2f} s, {t8:.2f} s): "
                       f"{c_row * 1e3:.1f} ms per row, {prep:.2f} s per head for selection and centroids; "
                       f"extrapolated to {w.BH} heads x {w.L} rows = {t_full:.0f} s per call (lower bound: "
                       f"the full oracle backward also accumulates dk and dv per row)"),
            "seconds_measured": t1 + t8}


def algorithmic_flops(w) -> float:
    """The method's FLOPs per call (all heads): exact blocks 4 L K B d, centroid scores
    2 L nblk d, zeroth order 2 L nU d, first order 2 L nU d^2 (order >= 1) and the exact
    second-order mass 2 L nU d^2 (order 2), nU = nblk - K."""
    nU = w.nblk - w.K
    f = 4.0 * w.L * w.K * w.B * w.d + 2.0 * w.L * w.nblk * w.d + 2.0 * w.L * nU * w.d
    if w.order >= 1:
        f += 2.0 * w.L * nU * w.d * w.d
    if w.order == 2:
        f += 2.0 * w.L * nU * w.d * w.d
    return f * w.BH


def stc_executed_flops(w, mask) -> float:
    """FLOPs the statistics-form tensor-core kernel executes for this selection: per CTA of
    256 rows, its union U of the selected blocks of its query tiles runs in 128-key tiles
    (S and PV: 4 d 128 per row and tile), every other block in items of g blocks (one MMA
    with N = g d + 16 per row: 2 d (g d + 16)), g = 2 for d = 64 and 1 for d = 128."""
    nu = cta_unions(w, mask)
    bpt, gb = 128 // w.B, (2 if w.d == 64 else 1)
    nut = (nu + bpt - 1) // bpt
    ni = (w.nblk - nu + gb - 1) // gb
    per_row = 4.0 * w.d * 128 * nut + 2.0 * w.d * (gb * w.d + 16) * ni
    return float(256.0 * per_row.sum())


def cta_unions(w, mask):
    """Per (bh, 256-row CTA): the number of blocks selected by any of its query tiles."""
    m = mask.cpu().numpy().view(np.uint32)  # [BH, nblk, words]
    BH, nblk, words = m.shape
    nqt = 256 // w.B
    ncta = (w.L + 255) // 256
    pad = ncta * nqt - nblk
    if pad > 0:
        # rows past L repeat the last tile's selection (the kernels clamp the tile index)
        m = np.concatenate([m, np.repeat(m[:, -1:], pad, axis=1)], axis=1)
    u = np.bitwise_or.reduce(m.reshape(BH, ncta, nqt, words), axis=2)
    return np.unpackbits(u.view(np.uint8), axis=-1).reshape(BH, ncta, -1).sum(axis=-1).astype(np.int64)


def hybrid_executed_flops(w, mask) -> float:
    """FLOPs the hybrid kernel executes for this selection: per 256-row CTA, its union tiles
    and the ceil(nblk/128) virtual tiles (S and PV: 4 d 128 per row and tile), plus the
    epilogue's G = Q H-bar^T (2 d^2 per row, order >= 1)."""
    nu = cta_unions(w, mask)
    bpt = 128 // w.B
    tiles = (nu + bpt - 1) // bpt + (w.nblk + 127) // 128
    per_row = 4.0 * w.d * 128 * tiles + (2.0 * w.d * w.d if w.order >= 1 else 0.0)
    return float(256.0 * per_row.sum())


def stats_bytes(w, order, es, kaug) -> float:
    """Compulsory HBM bytes of the statistics kernel: read K and V, write kbar and vsum
    (fp32), H_j (and C_j for order 2) in the input dtype, and the bf16 centroid split."""
    b = 2.0 * w.BH * w.L * w.d * es + 2.0 * w.BH * w.nblk * w.d * 4
    b += w.BH * w.nblk * w.d * w.d * es * (2 if order == 2 else 1)
    if kaug:
        b += w.BH * w.nblk * 8 * w.d * 2
    return b


def describe(w) -> str:
    """One-line description of a named workload (its shape and generator)."""
    shape = {"c3": "Wan2.1-shaped DiT attention", "c4": "Hunyuan-Video-shaped DiT attention"}.get(w.name)
    if w.kind == "field3d":
        gen = "x".join(str(g) for g in w.grid) + " video grid"
        shape = shape or "video-shaped attention"
    elif w.kind == "image_text":
        gen = "x".join(str(g) for g in w.grid) + f" image grid + {w.text_tokens} text tokens"
        shape = "FLUX-shaped image attention"
    else:
        gen = f"{w.n_centres} cluster centres"
        shape = "clustered-key attention"
    return (f"{w.name}: {shape}, batch 1 x {w.BH} heads, L={w.L} ({gen}), d={w.d}, B={w.B}, K={w.K}, "
            f"order={w.order}, {w.dtype}")


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, on the same workload/metric."""
    import pisa_synth

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = pisa_synth.workloads()[args.workload]
    q, k, v = pisa_synth.generate(w.with_(heads=1))
    times = []
    base = None
    for _ in range(args.warmup + args.steps):
        r = cpu_baseline(w, q, k, v)
        r.pop("_ref", None)
        times.append(r)
        base = r
    vals = [r["value"] for r in times[args.warmup:]] or [base["value"]]
    val = statistics.median(vals)
    ms = 4.0 * w.L * w.L * w.d * w.BH / (val * 1e12) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(w), "l2": "n/a (CPU)"},
        "cpu_baseline": {"kind": base["kind"], "cores": base["cores"], "sample": base["sample"], "value": val,
                         "unit": UNIT},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if world_plan(args.gpus, os.environ) == "launch":
        sys.exit(launch_ranks(args.gpus))
    if args.impl == "reference":
        run_reference(args)
        return
    import torch

    import block_sparse_taylor_b200 as pisa
    import pisa_synth

    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    w_all = pisa_synth.workloads()[args.workload]
    if args.heads:
        w_all = w_all.with_(heads=args.heads)
    tdt = torch.bfloat16 if w_all.dtype == "bf16" else torch.float32
    sharded = world > 1 and args.shard == "heads"
    if sharded:
        # one workload, its (batch, head) units split across the ranks: rank 0 draws the
        # inputs once and broadcasts them (before anything is timed); each rank keeps its slice
        from block_sparse_taylor_b200 import shard

        u0, u1 = shard.unit_range(w_all.BH, world, rank)
        full = []
        if rank == 0:
            q_h, k_h, v_h = pisa_synth.generate(w_all)
            full = [torch.from_numpy(x).to(tdt).cuda() for x in (q_h, k_h, v_h)]
        else:
            q_h = k_h = v_h = None
            full = [torch.empty((w_all.BH, w_all.L, w_all.d), dtype=tdt, device="cuda") for _ in range(3)]
        import torch.distributed as dist

        for t in full:
            dist.broadcast(t, src=0)
        q, k, v = (t[u0:u1].clone() for t in full)
        del full
        torch.cuda.synchronize()
        w = w_all.with_(heads=u1 - u0, batch=1)
    else:
        # one rank, or weak scaling: every rank draws its own inputs of the whole workload
        u0, u1 = 0, w_all.BH
        w = rank_workload(w_all, rank)
        q_h, k_h, v_h = pisa_synth.generate(w)
        q = torch.from_numpy(q_h).to(tdt).cuda()
        k = torch.from_numpy(k_h).to(tdt).cuda()
        v = torch.from_numpy(v_h).to(tdt).cuda()
    BH, L, d, B, K, order = w.BH, w.L, w.d, w.B, w.K, w.order
    nblk = L // B
    path = pisa.pisa_resolve_path(1, BH, L, d, B, K, order, tdt)
    out = torch.empty_like(q)
    kbar = torch.empty((BH, nblk, d), dtype=torch.float32, device="cuda")
    words = (nblk + 31) // 32
    idx = torch.empty((BH, nblk, K), dtype=torch.int32, device="cuda")
    mask = torch.empty((BH, nblk, words), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    stats_full = None
    stats_order = 1 if path == "stats_tc" else order  # the tensor-core statistics form reads H_j only
    if path in ("stats", "stats_tc"):
        stats_full = pisa.pisa_stats(k, v, B, stats_order)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if path in ("stats", "stats_tc"):
            st = pisa.pisa_stats(k, v, B, stats_order, buf=stats_full.buf)
        else:
            st = pisa.pisa_centroids(k, B, kbar=kbar)
        if ev is not None:
            ev[1].record(stream)
        lib = pisa.lib()
        pisa._check(lib.pisa_select(q.data_ptr(), pisa.ctypes.byref(st.raw), K, idx.data_ptr() if K else None,
                                    mask.data_ptr(), stream.cuda_stream))
        if ev is not None:
            ev[2].record(stream)
        pisa.pisa_fused_attention(q, k, v, B, mask, order, path=path, stats=st if path != "recompute_tc" else None,
                                  out=out)
        if ev is not None:
            ev[3].record(stream)

    # inputs smaller than twice the 126 MB L2 get an L2 flush (a 512 MiB write)
    # before every timed step, outside that step's events
    big_inputs = 3 * q.numel() * q.element_size() > 2 * 126 * 2 ** 20
    flush = None if big_inputs else torch.empty(512 * 2 ** 20, dtype=torch.uint8, device="cuda")

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    pisa.pisa_poll_device_status()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        if flush is not None:
            flush.zero_()
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    pisa.pisa_poll_device_status()
    total_ms = t_start.elapsed_time(t_end)
    if flush is not None:
        # the flushes sit between the steps: sum the steps' own spans
        total_ms = sum(e[0].elapsed_time(e[3]) for e in evs)
    total_ms = max_over_ranks(total_ms, world)
    ms_step = total_ms / args.steps
    k_prep = [e[0].elapsed_time(e[1]) for e in evs]
    k_sel = [e[1].elapsed_time(e[2]) for e in evs]
    k_attn = [e[2].elapsed_time(e[3]) for e in evs]
    attn_ms = statistics.mean(k_attn)
    step_spans = sorted(e[0].elapsed_time(e[3]) for e in evs)  # this rank's per-step spans
    step_pct = {"p10": pct(step_spans, 10), "median": pct(step_spans, 50), "p90": pct(step_spans, 90)}

    dense_flops = 4.0 * L * L * d * BH  # this rank's share
    # the whole job: every unit of the workload once (head-sharded), or one workload per rank
    job_flops = 4.0 * L * L * d * w_all.BH if sharded else dense_flops * world
    value = job_flops / (ms_step * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    if path in ("recompute_tc", "stats_tc"):
        # achieved = the method's algorithmic FLOPs (exact blocks, centroid scores,
        # zeroth- and first-order terms) per launch over the kernel's event time;
        # the FLOPs of the association actually executed are reported beside them
        alg_flops = algorithmic_flops(w)
        if path == "recompute_tc":
            exec_flops = 4.0 * L * L * d * BH  # QK^T and PV over every key block
            kname = f"attn_tc_kernel<{d},{B},{order}>"
        else:
            exec_flops = stc_executed_flops(w, mask)
            kname = f"attn_stc_kernel<{d},{B},{order}>"
        achieved = alg_flops / (attn_ms * 1e-3) / 1e12
        peak = float(peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic_record(w.name) if (not args.heads and path == "recompute_tc") else None,
                "kernel": kname,
                "algorithmic_flops_per_launch": alg_flops,
                "executed_flops_per_launch": exec_flops,
                "executed_tflops": exec_flops / (attn_ms * 1e-3) / 1e12,
                "executed_frac": exec_flops / (attn_ms * 1e-3) / 1e12 / peak,
                "peak_source": f"{peak_kind} bf16 dense (burst; the kernel is timed alone inside the step)"}
    else:
        # statistics path: CUDA-core kernel; report against the HBM roofline of its reads
        nbytes = 3 * BH * L * d * q.element_size()
        achieved = nbytes / (attn_ms * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": None, "kernel": f"attn_stats_kernel<{d},{B}>", "peak_source": peak_kind}
    # HBM figures of the small kernels (centroids read K once, or the statistics
    # kernel reads K and V and writes the statistics; select reads Q once + writes the mask)
    es = q.element_size()
    if path in ("stats", "stats_tc"):
        prep_bytes = stats_bytes(w, stats_order, es, kaug=(path == "stats_tc"))
        prep_name = ("stats_tc_kernel" if tdt == torch.bfloat16 else "stats_simt_kernel") + f"<{d},{B},{stats_order}>"
    else:
        prep_bytes = BH * L * d * es + BH * nblk * d * 4
        prep_name = f"centroid_kernel<{d},{B}>"
    sel_bytes = BH * L * d * es + BH * nblk * (words + K) * 4
    hbm = float(peaks["hbm_gbs"])
    per_kernel = {
        "prep_kernel": prep_name,
        "centroids_ms": statistics.mean(k_prep), "select_ms": statistics.mean(k_sel), "attn_ms": attn_ms,
        "centroids_gbs": prep_bytes / (statistics.mean(k_prep) * 1e-3) / 1e9,
        "select_gbs": sel_bytes / (statistics.mean(k_sel) * 1e-3) / 1e9,
    }
    per_kernel["centroids_frac_hbm"] = per_kernel["centroids_gbs"] / hbm
    per_kernel["select_frac_hbm"] = per_kernel["select_gbs"] / hbm

    # The statistics kernel (block statistics k-bar, v-sum, H_j and, for order 2,
    # C_j) is not on the token-form path; it is timed here on its own against
    # the HBM roofline of its compulsory traffic.
    stats_rec = None
    if path not in ("stats", "stats_tc"):
        sorder = max(order, 1)
        sbuf = torch.empty(pisa.pisa_stats_bytes(1, BH, L, d, B, sorder, tdt), dtype=torch.uint8, device="cuda")
        for _ in range(2):
            pisa.pisa_stats(k, v, B, sorder, buf=sbuf)
        sa, sb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        sa.record(stream)
        for _ in range(reps):
            pisa.pisa_stats(k, v, B, sorder, buf=sbuf)
        sb.record(stream)
        torch.cuda.synchronize()
        s_ms = sa.elapsed_time(sb) / reps
        s_bytes = stats_bytes(w, sorder, es, kaug=(tdt == torch.bfloat16))
        kname = "stats_tc_kernel" if tdt == torch.bfloat16 else "stats_simt_kernel"
        stats_rec = {"kernel": f"{kname}<{d},{B},{sorder}>", "order": sorder, "ms": s_ms,
                     "algorithmic_bytes": s_bytes, "gbs": s_bytes / (s_ms * 1e-3) / 1e9,
                     "frac_hbm": s_bytes / (s_ms * 1e-3) / 1e9 / hbm}
        del sbuf

    # Covariance-aware routing (opt-in): the bias kernel ln(||H_j||_F + eps) and
    # the biased selection, timed on their own on the same inputs.
    route_rec = None
    if path != "stats" and not args.no_route:
        # its own selection buffers: the timed step's mask stays for the parity record
        idx_rt = torch.empty_like(idx)
        mask_rt = torch.empty_like(mask)
        rb = torch.empty((BH, nblk), dtype=torch.float32, device="cuda")
        st_c = pisa.pisa_centroids(k, B, kbar=kbar)
        for _ in range(2):
            pisa.pisa_route_bias(k, v, kbar, B, out=rb)
        ra, rb_ev, rc_ev = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        reps = 5
        ra.record(stream)
        for _ in range(reps):
            pisa.pisa_route_bias(k, v, kbar, B, out=rb)
        rb_ev.record(stream)
        for _ in range(reps):
            pisa._check(pisa.lib().pisa_select_biased(q.data_ptr(), pisa.ctypes.byref(st_c.raw), K,
                                                       rb.data_ptr(), idx_rt.data_ptr() if K else None,
                                                       mask_rt.data_ptr(), stream.cuda_stream))
        rc_ev.record(stream)
        torch.cuda.synchronize()
        pisa.pisa_poll_device_status()
        r_ms = ra.elapsed_time(rb_ev) / reps
        route_rec = {"bias_kernel": f"route_bias_kernel<{d},{B}>", "bias_ms": r_ms,
                     "bias_gflops_fp32": 2.0 * BH * nblk * B * d * d / (r_ms * 1e-3) / 1e9,
                     "select_biased_ms": rb_ev.elapsed_time(rc_ev) / reps,
                     "note": "scalar IEEE fp32 in a canonical order (reproducible bit for bit), CUDA cores"}
        del rb, idx_rt, mask_rt

    # The PISA hybrid (global H-bar, the paper's own speed path) on the same
    # inputs: a separate record, timed as whole calls of pisa_attention.
    hybrid_rec = None
    if not args.no_hybrid and tdt == torch.bfloat16 and order <= 1:
        hws = torch.empty(pisa.pisa_workspace_bytes(1, BH, L, d, B, K, order, tdt, "hybrid_tc"), dtype=torch.uint8,
                          device="cuda")
        hout = torch.empty_like(q)
        for _ in range(3):
            pisa.pisa_attention(q, k, v, B, K, order, path="hybrid_tc", out=hout, workspace=hws)
        ha, hb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(5, args.steps)
        ha.record(stream)
        for _ in range(reps):
            pisa.pisa_attention(q, k, v, B, K, order, path="hybrid_tc", out=hout, workspace=hws)
        hb.record(stream)
        torch.cuda.synchronize()
        pisa.pisa_poll_device_status()
        h_ms = ha.elapsed_time(hb) / reps
        h_exec = hybrid_executed_flops(w, mask)
        bf16_peak = float(peaks["bf16_tflops"])
        hybrid_rec = {"method": "PISA hybrid: exact selected blocks, zeroth-order virtual tokens, global H-bar "
                                "first-order term (not the per-block H_j formulation of the main line)",
                      "ms_per_call": h_ms, "full_attn_equiv_tflops": dense_flops / (h_ms * 1e-3) / 1e12,
                      "speedup_vs_per_block_path": ms_step / h_ms, "launches_per_call": 5,
                      "roofline": {"bound": "tensor", "kernel": f"attn_hybrid_kernel<{d},{B},{order}>",
                                   "executed_flops_per_call": h_exec,
                                   "achieved": h_exec / (h_ms * 1e-3) / 1e12, "peak": bf16_peak,
                                   "unit": "TFLOP/s", "frac": h_exec / (h_ms * 1e-3) / 1e12 / bf16_peak,
                                   "note": "executed FLOPs of the attention kernel (union tiles, virtual tiles, "
                                           "Q H-bar^T) over the whole call's time (prepare, select, attention): a "
                                           "lower bound on the attention kernel's own fraction",
                                   "peak_source": f"{peak_kind} bf16 dense (burst)"}}
        del hws, hout

    # The backward pass (training use) on the same inputs: dq, dk, dv of
    # sum(dO * o) for the forward output o above, selection held fixed; timed
    # as whole calls (centroids, selection, delta, dq, dk/dv) given the
    # forward's log-denominators, as the autograd function calls it.
    bwd_rec = None
    if not args.no_backward:
        gen = torch.Generator(device="cuda").manual_seed(4321 + rank)
        dO = torch.randn(q.shape, generator=gen, device="cuda", dtype=torch.float32).to(tdt)
        grads = tuple(torch.empty(q.shape, dtype=torch.float32, device="cuda") for _ in range(3))
        bws = torch.empty(pisa.pisa_backward_workspace_bytes(1, BH, L, d, B, K, order, tdt), dtype=torch.uint8,
                          device="cuda")
        _, lse = pisa.pisa_attention_lse(q, k, v, B, K, order)
        for _ in range(2):
            pisa.pisa_attention_backward(q, k, v, out, dO, B, K, order, grads=grads, workspace=bws, lse=lse)
        torch.cuda.synchronize()
        pisa.pisa_poll_device_status()
        ba, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        ba.record(stream)
        for _ in range(reps):
            pisa.pisa_attention_backward(q, k, v, out, dO, B, K, order, grads=grads, workspace=bws, lse=lse)
        bb.record(stream)
        torch.cuda.synchronize()
        pisa.pisa_poll_device_status()
        b_ms = ba.elapsed_time(bb) / reps
        tc_bwd = tdt == torch.bfloat16 and d in (64, 128) and B in (64, 128) and L % 128 == 0
        alg = 10.0 * L * L * d * BH       # S, dP, dq, dk, dv once each (five products of 2 L^2 d)
        # tcgen05 path: S, G, dQ in the dq kernel and S, G, dK, dV in the dk/dv kernel
        executed = (14.0 if tc_bwd else 16.0) * L * L * d * BH
        bf16_peak = float(peaks["bf16_tflops"])
        kernels = ([f"bwd_delta_kernel<{d}>", f"bwd_dq_tc_kernel<{d},{B},{order}>",
                    f"bwd_dkdv_tc_kernel<{d},{B},{order}>"] if tc_bwd else
                   [f"bwd_rowstat_kernel<{d},{B}>", f"bwd_dq_kernel<{d},{B}>", f"bwd_dkdv_kernel<{d},{B}>"])
        bwd_rec = {"kernels": kernels,
                   "ms_per_call": b_ms, "algorithmic_flops_per_call": alg,
                   "algorithmic_tflops": alg / (b_ms * 1e-3) / 1e12,
                   "executed_tflops": executed / (b_ms * 1e-3) / 1e12,
                   "roofline": ({"bound": "tensor", "peak": bf16_peak, "unit": "TFLOP/s",
                                 "frac": alg / (b_ms * 1e-3) / 1e12 / bf16_peak,
                                 "frac_executed": executed / (b_ms * 1e-3) / 1e12 / bf16_peak,
                                 "peak_source": f"{peak_kind} bf16 dense (burst)"}
                                if tdt == torch.bfloat16 else None),
                   "tile_products": ("tcgen05 128xN tiles, bf16 operands, fp32 accumulation in TMEM" if tc_bwd else
                                     "warp-level mma.sync m16n8k16, bf16 operands, fp32 accumulation"
                                     if tdt == torch.bfloat16 else "fp32 FMA"),
                   "lse": "from the forward (pisa_attention_lse)",
                   "launches_per_call": 5}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            try:
                bwd_rec["cpu_baseline"] = cpu_backward_baseline(w, q_h, k_h, v_h, dO[:1].float().cpu().numpy())
            except Exception as e:  # noqa: BLE001 - a baseline record never fails the benchmark
                bwd_rec["cpu_baseline"] = {"unavailable": f"{type(e).__name__}: {e}"[:240]}
        del dO, grads, bws, lse

    # end to end through the public host-buffer call: pisa_attention_host on
    # pinned host q, k, v, out (per chunk of heads: H2D copies, the attention,
    # D2H copy; two streams so that the copies overlap the kernels)
    e2e = None
    if not args.no_e2e:
        hq = q.cpu().pin_memory()
        hk = k.cpu().pin_memory()
        hv = v.cpu().pin_memory()
        ho = torch.empty_like(hq).pin_memory()
        plan = pisa.HostPlan(hq, B, K, order, chunk_heads=max(1, BH // 20))

        def e2e_step():
            for st_ in plan.streams:
                st_.wait_stream(stream)
            pisa.pisa_attention_host(hq, hk, hv, ho, plan)
            for st_ in plan.streams:
                stream.wait_stream(st_)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_ms = max_over_ranks(a.elapsed_time(b) / args.steps, world)
        job_units = w_all.BH if sharded else BH * world
        unit_bytes = L * d * q.element_size()
        e2e = {"value": job_flops / (e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": 3 * job_units * unit_bytes,
               "d2h_bytes_per_step": job_units * unit_bytes,
               "call": f"pisa_attention_host, {plan.chunk} heads per chunk, two streams"}
        pisa.pisa_poll_device_status()
        del plan

    dense_rec = None
    if not args.no_dense and rank == 0 and world == 1:
        dense_rec = dense_sdpa_record(q, k, v, stream)
        if "ms_per_call" in dense_rec:
            dense_rec["speedup_of_pisa_step"] = dense_rec["ms_per_call"] / ms_step

    cpu = None
    par = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, q_h, k_h, v_h)
        try:
            par = parity_record(w, out, mask, q_h, k_h, cpu.pop("_ref"))
        except Exception as e:  # noqa: BLE001 - reported, never raised
            par = {"unavailable": f"{type(e).__name__}: {e}"[:240]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": describe(w_all),
                       "path": path, "global_batch": 1 if sharded else world, "seq_len": L,
                       "parallelism": (f"heads sharded over {world} ranks (rank 0: units {u0}..{u1 - 1} of "
                                       f"{w_all.BH}; no data-path collective)" if sharded else
                                       f"replicas x{world} (heads independent, no collective)"),
                       "l2": ("inputs exceed L2 (3 x {:.0f} MiB per rank), no flush" if big_inputs else
                              "inputs fit in L2 (3 x {:.0f} MiB per rank); L2 flushed before every step").format(
                           q.numel() * q.element_size() / 2 ** 20)},
            "roofline": roof,
            "per_kernel": per_kernel,
            "stats_kernel": stats_rec,
            "hybrid": hybrid_rec,
            "routing": route_rec,
            "backward": bwd_rec,
            "step_ms_percentiles": step_pct,
            "dense_sdpa_context": dense_rec,
            "cpu_baseline": cpu,
            "parity": par,
            "clocks": clk,
            "e2e": e2e,
            "gpu_launches": 3 * args.steps,
            "tflops_executed_attn": roof["achieved"] if roof["unit"] == "TFLOP/s" else None,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
