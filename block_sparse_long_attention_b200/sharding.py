"""Split a global batch of independent (batch, head) problems over ranks.

BigBird attention of different sequences and heads is independent, so a
multi-GPU run gives each rank a contiguous slice of the batch and exchanges
nothing on the data path.
"""

from __future__ import annotations


def batch_shard(global_batch: int, world: int, rank: int) -> tuple[int, int]:
    """[lo, hi) of the sequences rank `rank` of `world` owns; balanced, contiguous."""
    if world <= 0 or not 0 <= rank < world or global_batch < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(global_batch, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)
