"""Multi-process host logic on CPU (gloo, world size 2).

The path shards by (batch, head) with no data-path collective.  Head-sharded
(the default of bench.py on several GPUs): rank r computes a contiguous slice
of one call's units with the unchanged single-GPU call, and an optional
all-gather reassembles the output; here the per-rank compute is the CPU oracle
and the test checks that the slices reassemble to the unsharded result bit for
bit.  Replicas: every rank runs the whole workload on its own inputs (weak
scaling).  The timing barrier and the max-over-ranks reduction of the elapsed
time run here on gloo ranks too.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import pisa_synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        local_ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(local_ms, world, device="cpu")
        w = pisa_synth.workloads()["c1"]
        wr = bench.rank_workload(w, rank)
        qh, _, _ = pisa_synth.generate(wr)
        digest = float(np.abs(qh).sum())
        t = torch.tensor([digest], dtype=torch.float64)
        gathered = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(gathered, t)
        q.put((rank, mx, [float(g.item()) for g in gathered]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_timing_and_weak_scaling_inputs():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=100) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, mx, digests in res:
        assert mx == 15.0  # every rank reports the slowest rank's time
        assert digests[0] != digests[1]  # each replica draws its own inputs


def test_rank_zero_keeps_the_canonical_seed():
    import bench

    w = pisa_synth.workloads()["c3"]
    assert bench.rank_workload(w, 0) == w
    assert bench.rank_workload(w, 3).seed != w.seed


def _shard_worker(rank, world, port, q, BH):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    from block_sparse_taylor_b200 import shard

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        qq, kk, vv = pisa_synth.random_qkv(4242, BH, 512, 64, scale=2.0)
        u0, u1 = shard.unit_range(BH, world, rank)
        # this rank's share of the units, computed alone (the oracle stands in for the GPU call)
        local = torch.from_numpy(oracle.pisa_attention(qq[u0:u1], kk[u0:u1], vv[u0:u1], 64, 2, 1, nthreads=2))
        total = shard.total_units(local.shape[0])
        full = shard.gather_units(local, total)
        view = shard.local_units(torch.from_numpy(qq), world, rank)
        q.put((rank, (u0, u1), total, full.numpy(), bool(np.array_equal(view.numpy(), qq[u0:u1]))))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("BH", [4, 5])
def test_head_shards_reassemble_to_the_unsharded_call(BH):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q, BH)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=150) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    qq, kk, vv = pisa_synth.random_qkv(4242, BH, 512, 64, scale=2.0)
    want = oracle.pisa_attention(qq, kk, vv, 64, 2, 1)
    ranges = [r[1] for r in res]
    assert ranges[0][0] == 0 and ranges[0][1] == ranges[1][0] and ranges[1][1] == BH  # a partition
    for rank, rng_, total, full, view_ok in res:
        assert total == BH and view_ok
        assert np.array_equal(full, want)  # every rank holds the whole output, bit for bit


def test_unit_ranges_partition_the_units():
    from block_sparse_taylor_b200 import shard

    for units in (1, 3, 5, 24, 40, 41):
        for world in (1, 2, 3, 8):
            if world > units:
                continue
            r = [shard.unit_range(units, world, k) for k in range(world)]
            assert r[0][0] == 0 and r[-1][1] == units
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [b - a for a, b in r]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.unit_range(4, 2, 2)


def test_bench_starts_or_refuses_ranks_to_match_gpus():
    import bench

    assert bench.world_plan(1, {}) == "run"
    assert bench.world_plan(8, {}) == "launch"  # no torchrun around it: bench.py starts 8 ranks
    assert bench.world_plan(8, {"WORLD_SIZE": "8"}) == "run"
    with pytest.raises(SystemExit):
        bench.world_plan(8, {"WORLD_SIZE": "1"})  # never report n_gpus 1 for --gpus 8
    with pytest.raises(SystemExit):
        bench.world_plan(0, {})
