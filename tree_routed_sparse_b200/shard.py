"""Partition of the independent (b, h) problems of one batch across ranks.

Every (batch, head) pair owns its tree and its queries and no step reads another pair's data, so
a batch divides across GPUs without any data-path collective: rank k processes a contiguous
range of flat block indices b*H + h.

A weak-scaling run on `world` GPUs processes a global batch of world times the per-GPU
sequences; every rank draws only its own blocks from the seeded generator (each element at its
flat index in the global batch), so the shards of one run are disjoint parts of one batch.
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


def global_workload(wl, world: int):
    """The global batch of a weak-scaling run: `world` times the per-GPU sequences."""
    if world < 1:
        raise ValueError(f"world {world}")
    return wl.replace(batch=wl.batch * world)


def shard_inputs(wl_global, world: int, rank: int, device="cpu") -> tuple[int, int, dict]:
    """(lo, hi, inputs) of `rank`'s blocks [lo, hi) of the global batch; the inputs are shaped
    [sequences, heads, ...] when the range is whole sequences, else [1, hi - lo, ...]."""
    from . import synth
    lo, hi = shard_range(wl_global.bh, world, rank)
    inp = synth.make_block_inputs(wl_global, lo, hi, device)
    H = wl_global.heads
    if lo % H == 0 and hi % H == 0:
        inp = synth.as_sequences(inp, H)
    return lo, hi, inp
