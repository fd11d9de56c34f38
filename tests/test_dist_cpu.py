"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The path shards by (batch, head) with no data-path collective: every rank runs
its own replica of the workload on its own inputs (weak scaling).  The only
collective steps are the timing barrier and the max-over-ranks reduction of
the elapsed time; these run here on gloo ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

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
