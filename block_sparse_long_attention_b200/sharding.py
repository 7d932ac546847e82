"""Split independent (batch, head) problems over ranks.

BigBird attention of different sequences and heads is independent, so a
multi-GPU run gives each rank a contiguous slice of the batch (the benchmark:
nothing is exchanged on the data path) or of the heads (sharded_fwd, for B*H
too large for one GPU: the only exchange is the optional all-gather of the
output along the head axis).
"""

from __future__ import annotations


def batch_shard(global_batch: int, world: int, rank: int) -> tuple[int, int]:
    """[lo, hi) of the sequences rank `rank` of `world` owns; balanced, contiguous."""
    if world <= 0 or not 0 <= rank < world or global_batch < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(global_batch, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def head_shard(H: int, world: int, rank: int) -> tuple[int, int]:
    """[lo, hi) of the heads rank `rank` of `world` owns; balanced, contiguous."""
    return batch_shard(H, world, rank)


def sharded_fwd(q, k, v, rand_attn, seq_mask=None, *, block: int = 64, r: int = 3, group=None, gather: bool = True,
                compute=None):
    """Head-sharded forward over a torch.distributed process group.

    Every rank passes the full-shape inputs it has (only its own heads are
    read): rank i of the group computes heads head_shard(H, world, i) of every
    sequence -- rand_attn is per head, so each rank takes its rows of it --
    and, with gather=True, the outputs are all-gathered along the head axis
    (NCCL over NVLink on GPUs). Heads are independent: the gather is the only
    exchange. Returns the full [B, H, L, d] output (gather=True) or this
    rank's [B, hi-lo, L, d] slice.

    compute(q, k, v, rand_attn, seq_mask, block, r) defaults to the CUDA
    forward (bigbird_attn_fwd through the package's fwd()).
    """
    import torch
    import torch.distributed as dist

    if compute is None:
        from . import fwd as _fwd

        def compute(q_, k_, v_, ra_, sm_, block_, r_):
            return _fwd(q_, k_, v_, ra_, sm_, block=block_, r=r_)
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    B, H, L, d = q.shape
    lo, hi = head_shard(H, world, rank)
    sl = slice(lo, hi)
    part = compute(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(),
                   None if rand_attn is None else rand_attn[sl].contiguous(), seq_mask, block, r)
    if not gather or world == 1:
        return part
    # all_gather needs equal shapes: pad every rank's slice to the largest shard
    maxh = max(b - a for a, b in (head_shard(H, world, i) for i in range(world)))
    buf = torch.zeros((B, maxh, L, d), dtype=part.dtype, device=part.device)
    buf[:, : hi - lo] = part
    bufs = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(bufs, buf, group=group)
    pieces = [g[:, : b - a] for g, (a, b) in zip(bufs, (head_shard(H, world, i) for i in range(world)))]
    return torch.cat(pieces, dim=1)
