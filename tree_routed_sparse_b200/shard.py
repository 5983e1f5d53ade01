"""Partition of the independent (b, h) problems of one batch across ranks.

Every (batch, head) pair owns its tree and its queries and no step reads another pair's data, so
a batch divides across GPUs without any data-path collective: rank k processes a contiguous
range of flat block indices b*H + h.
"""
from __future__ import annotations


def shard_range(total: int, world: int, rank: int) -> tuple[int, int]:
    """[lo, hi) of the flat blocks owned by `rank`: contiguous, sizes differing by at most one."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError(f"bad shard request total={total} world={world} rank={rank}")
    base, rem = divmod(total, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)


def blocks_of(batch: int, heads: int, world: int, rank: int) -> list[tuple[int, int]]:
    """The (b, h) pairs owned by `rank`, in flat order."""
    lo, hi = shard_range(batch * heads, world, rank)
    return [divmod(k, heads) for k in range(lo, hi)]
