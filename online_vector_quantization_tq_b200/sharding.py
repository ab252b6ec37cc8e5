"""Multi-GPU sharding of the scoring path (one process per GPU).

Encode and KV scoring shard by key with no exchange: each rank owns a
contiguous range of keys (or whole KV heads) and writes its own outputs.
Top-k retrieval over a database sharded by rows has one exchange: every rank
finds the top-k of its own rows (tq_topk, global row indices), the ranks
all-gather those k candidates per query (q x k scores and indices, a few KB),
and each rank merges them.  The merge keeps the library's order: descending
score, equal scores by ascending row index.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [lo, hi) share of n rows for `rank` (sizes differ by <= 1)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def merge_topk(scores: torch.Tensor, idx: torch.Tensor, k: int) -> tuple[torch.Tensor, torch.Tensor]:
    """Top-k over candidate columns: descending score, then ascending index."""
    # sort by index first, then stably by score, so equal scores keep index order
    o1 = torch.argsort(idx, dim=1, stable=True)
    s1 = torch.gather(scores, 1, o1)
    i1 = torch.gather(idx, 1, o1)
    o2 = torch.argsort(s1, dim=1, descending=True, stable=True)
    return torch.gather(s1, 1, o2)[:, :k], torch.gather(i1, 1, o2)[:, :k]


def allgather_topk(local_scores: torch.Tensor, local_idx: torch.Tensor, k: int, group=None):
    """Global top-k from every rank's local top-k (same shape on all ranks;
    empty slots carry score -inf and index -1)."""
    world = dist.get_world_size(group)
    gs = [torch.empty_like(local_scores) for _ in range(world)]
    gi = [torch.empty_like(local_idx) for _ in range(world)]
    dist.all_gather(gs, local_scores.contiguous(), group=group)
    dist.all_gather(gi, local_idx.contiguous(), group=group)
    return merge_topk(torch.cat(gs, dim=1), torch.cat(gi, dim=1), k)


def max_over_ranks(values: list[float], device=None, group=None) -> list[float]:
    """Element-wise maximum over ranks (the timing rule for multi-GPU runs)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t.tolist()
