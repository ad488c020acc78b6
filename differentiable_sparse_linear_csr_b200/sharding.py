"""Splitting one batch of independent systems across ranks (one process per GPU).

Systems that share a pattern are independent (torch-sla summary page, technical
summary, "Methodology" 1: a SparseTensor batch shares one pattern; each system
is solved on its own), so a fixed batch of B systems shards along B with no
exchange during the solve: rank r solves systems [lo_r, hi_r) with the pattern
replicated on every GPU, and the per-rank results are gathered once afterwards
if a caller wants them in one place.  A single system does not shard this way
(it would need a halo exchange before every SpMV), so it is left to replicas.

Host-side bookkeeping only: the solve on each rank is the library's, and the
gather is one torch.distributed all_gather after it.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(total: int, world: int, rank: int) -> tuple[int, int]:
    """Systems [lo, hi) of rank `rank` out of `total`: contiguous, sizes differ
    by at most one, every system in exactly one shard (ranks beyond `total` get
    an empty range)."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError(f"shard_range: total={total}, world={world}, rank={rank}")
    return (rank * total) // world, ((rank + 1) * total) // world


def gather_shards(local: torch.Tensor, total: int, group=None) -> torch.Tensor:
    """The [total, ...] batch from every rank's [hi - lo, ...] shard, on every
    rank, in system order.  Shards of unequal size are padded for the
    collective and trimmed after it."""
    world = dist.get_world_size(group)
    sizes = [shard_range(total, world, r) for r in range(world)]
    width = max(hi - lo for lo, hi in sizes)
    pad = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([parts[r][:hi - lo] for r, (lo, hi) in enumerate(sizes)], dim=0)
