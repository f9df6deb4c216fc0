"""One long sequence's context split over ranks, one GPU each -- the path's one exchange step.

Each rank keeps a contiguous token range of every sequence in its own compressed cache (the decode
step appends the new token on the last rank) and attends over it with ``Cache.attend(partial=True)``:
per query head the log-sum-exp row (m, l, o[128]) of its range.  The rows of all ranks are
all-gathered -- 520 bytes per query head and rank -- and merged by ``kv1b_merge_partials``, the same
log-sum-exp merge that joins the split-K pieces inside one GPU, so the result equals the attention
over the whole context.  ``torch.distributed`` carries the exchange (NCCL between GPUs, gloo for host
tensors); nothing else crosses ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import merge_partials


def shard_bounds(length: int, world: int, rank: int) -> tuple[int, int]:
    """Token range [start, stop) of `rank` when `length` tokens are split into `world` contiguous,
    near-equal ranges (the first length % world ranks hold one token more)."""
    if world < 1 or not 0 <= rank < world or length < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, length >= 0")
    base, extra = divmod(length, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def append_rank(world: int) -> int:
    """The rank whose cache receives the decode step's new token (the last range grows)."""
    return world - 1


def exchange(part: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's partial rows: [world, *part.shape], rank r's rows at index r."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(part) for _ in range(world)]
    dist.all_gather(parts, part.contiguous(), group=group)
    return torch.stack(parts)


def attend(cache, q: torch.Tensor, scale: float, group=None, engine: int = 0) -> torch.Tensor:
    """Attention of q over the whole split context: this rank's partial rows, the exchange, the merge
    (on this rank's GPU).  Every rank of `group` calls it with the same q and gets the same output."""
    part = cache.attend(q, scale, engine=engine, partial=True)
    return merge_partials(exchange(part, group))
