"""Head-block sharding of one attention layer over ranks.

Every step of MC-Sparse works per (b, h) head: grouping, the exact
probabilities, the selection, the residual and the reused step never mix
heads (aiqbench.com, "MC-Sparse: Deconstructing and Closing the Dense-Sparse
Attention Gap in Diffusion Transformers", abstract: query groups, KV indices
and residuals are per attention head).  So one layer [B, H, N, d] shards over
W ranks with no exchange on the data path: rank r takes the contiguous block
of flattened heads bh = b*H + h in [start_r, start_r + count_r), the blocks'
sizes differing by at most one.  A block is a view of the layer at a pointer
offset (no copy): the library treats B*H as one axis, so the block is passed
as a layer of shape [1, count_r, N, d].

Collectives appear only outside the path: `gather_heads` reassembles a
sharded output for checks and reports.
"""
from __future__ import annotations

from typing import Tuple

import torch


def head_range(BH: int, world: int, rank: int) -> Tuple[int, int]:
    """(start, count) of rank `rank`'s contiguous block of the BH flattened
    heads: the first BH % world ranks take one head more."""
    if world < 1 or not 0 <= rank < world or BH < 0:
        raise ValueError(f"bad partition: BH={BH} world={world} rank={rank}")
    base, extra = divmod(BH, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def shard(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """Rank `rank`'s heads of a per-head tensor [B, H, ...] as a view
    [1, count, ...] (contiguous input, no copy)."""
    if not x.is_contiguous():
        raise ValueError("shard needs a contiguous [B, H, ...] tensor")
    B, H = x.shape[:2]
    start, count = head_range(B * H, world, rank)
    flat = x.view(B * H, *x.shape[2:])
    return flat.narrow(0, start, count).unsqueeze(0)


def gather_heads(local: torch.Tensor, BH: int, world: int, group=None) -> torch.Tensor:
    """All ranks' blocks [1, count_r, ...] concatenated in head order into
    [BH, ...] on every rank (torch.distributed all_gather; for checks and
    reports, not for the attention path)."""
    import torch.distributed as dist
    counts = [head_range(BH, world, r)[1] for r in range(world)]
    width = max(counts)
    tail = tuple(local.shape[2:])
    pad = torch.zeros((width, *tail), dtype=local.dtype, device=local.device)
    pad[:local.shape[1]] = local[0]
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)
