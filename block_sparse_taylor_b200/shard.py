"""Multi-GPU use: one call's (batch, head) units split across ranks.

Every (batch, head) unit of piecewise sparse attention is independent: its
statistics, selection and output read only that unit's q, k, v (PISA paper,
section 3.4 and Figure 3: the kernels run per (batch, head)).  So the work of
one call shards across GPUs by heads with no exchange on the data path: rank r
runs the unchanged single-GPU call on a contiguous slice of the units, and the
only collective is an optional all-gather of the outputs when a caller wants
the whole result on every rank.  Nothing here reads another GPU's memory.

The units are the folded leading axis of a [batch * heads, L, d] tensor (or
the first two axes of [batch, heads, L, d]); the split is contiguous and
balanced: the first (units % world) ranks take one unit more.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch


def unit_range(units: int, world: int, rank: int) -> Tuple[int, int]:
    """[u0, u1): the units rank ``rank`` of ``world`` computes."""
    if units <= 0 or world <= 0 or not 0 <= rank < world:
        raise ValueError(f"bad split: units={units}, world={world}, rank={rank}")
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    return u0, u0 + base + (1 if rank < extra else 0)


def _folded(x: torch.Tensor) -> torch.Tensor:
    if x.dim() == 4:
        return x.reshape(x.shape[0] * x.shape[1], x.shape[2], x.shape[3])
    if x.dim() == 3:
        return x
    raise ValueError("expected [batch, heads, L, d] or [batch*heads, L, d]")


def local_units(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """This rank's contiguous slice of the (batch, head) units, [u1 - u0, L, d] (a view)."""
    f = _folded(x)
    u0, u1 = unit_range(f.shape[0], world, rank)
    return f[u0:u1]


def gather_units(local: torch.Tensor, units: int, group=None) -> torch.Tensor:
    """All-gather the ranks' output slices (in rank order) into [units, L, d] on every rank.
    Slices of unequal size are padded to the largest for the collective and trimmed after."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    sizes = [unit_range(units, world, r) for r in range(world)]
    width = max(u1 - u0 for u0, u1 in sizes)
    rank = dist.get_rank(group)
    u0, u1 = sizes[rank]
    if local.shape[0] != u1 - u0:
        raise ValueError(f"rank {rank} holds {local.shape[0]} units, its share is {u1 - u0}")
    padded = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    padded[: local.shape[0]] = local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    return torch.cat([p[: b - a] for p, (a, b) in zip(parts, sizes)], dim=0)


def total_units(local_count: int, group=None) -> int:
    """The call's total number of units from every rank's local count (one all-reduce)."""
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([int(local_count)], dtype=torch.int64, device=dev)
    dist.all_reduce(t, group=group)
    return int(t.item())


def pisa_attention_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, B: int, K: int, order: int = 1,
                           group=None, gather: bool = False, units: Optional[int] = None,
                           out: Optional[torch.Tensor] = None, **kw):
    """Piecewise sparse attention of this rank's share of the (batch, head) units.

    q, k, v: the rank's slices, [u1 - u0, L, d] contiguous CUDA tensors (local_units of the
    full tensors).  Runs pisa_attention on them (same keyword options) and returns the local
    output, or with ``gather`` the whole [units, L, d] output on every rank (one all-gather
    over ``group``, NCCL for CUDA tensors; ``units`` is the total, counted if not given)."""
    from . import pisa_attention

    o = pisa_attention(q, k, v, B, K, order, out=out, **kw)
    if not gather:
        return o
    if units is None:
        units = total_units(o.shape[0], group)
    return gather_units(o, units, group)
