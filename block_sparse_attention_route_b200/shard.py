"""Head sharding of one BSA problem over ranks (one process per GPU).

Routing and attention of a head never read another head, so a batch splits over ranks by
heads with no exchange inside the path: each rank runs the pipeline on its head slice and,
if one rank needs the whole output, an all-gather over the head dimension assembles it.
"""
from __future__ import annotations

import dataclasses
from typing import Tuple


def head_range(rank: int, world: int, heads: int) -> Tuple[int, int]:
    """Contiguous [h0, h1) of this rank; the first heads % world ranks get one more head."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_geometry(g, rank: int, world: int):
    """The per-rank Geometry (same grid and blocks, this rank's head count)."""
    h0, h1 = head_range(rank, world, g.heads)
    return dataclasses.replace(g, heads=h1 - h0)


def gather_heads(local, heads: int, dim: int, group=None):
    """All-gather head slices (uneven splits allowed) along `dim` into the full tensor."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    sizes = [head_range(r, world, heads) for r in range(world)]
    width = max(h1 - h0 for h0, h1 in sizes)
    shape = list(local.shape)
    shape[dim] = width
    padded = torch.zeros(shape, dtype=local.dtype, device=local.device)
    padded.narrow(dim, 0, local.shape[dim]).copy_(local)
    bufs = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(bufs, padded, group=group)
    return torch.cat([b.narrow(dim, 0, h1 - h0) for b, (h0, h1) in zip(bufs, sizes)], dim=dim)
