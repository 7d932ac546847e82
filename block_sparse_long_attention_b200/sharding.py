"""Split independent (batch, head) problems over ranks.

BigBird attention of different sequences and heads is independent, so a
multi-GPU run gives each rank a contiguous slice of the batch
(batch_sharded_fwd; the benchmark's layout: nothing is exchanged on the data
path) or of the heads (sharded_fwd, for B*H too large for one GPU). In both
the only exchange is the optional all-gather of the output along the sharded
axis.
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


def _default_compute():
    from . import fwd as _fwd

    def compute(q_, k_, v_, ra_, sm_, block_, r_):
        return _fwd(q_, k_, v_, ra_, sm_, block=block_, r=r_)
    return compute


def _group_info(group):
    import torch.distributed as dist
    if not dist.is_initialized():
        return 1, 0, False
    return dist.get_world_size(group), dist.get_rank(group), True


def _all_gather_along(part, dim: int, shards, group):
    """All-gather every rank's slice along `dim` (slices may differ by one:
    each is padded to the largest so every rank sends the same shape) and
    concatenate them in rank order."""
    import torch
    import torch.distributed as dist
    maxn = max(b - a for a, b in shards)
    shape = list(part.shape)
    shape[dim] = maxn
    buf = torch.zeros(shape, dtype=part.dtype, device=part.device)
    buf.narrow(dim, 0, part.shape[dim]).copy_(part)
    bufs = [torch.empty_like(buf) for _ in shards]
    dist.all_gather(bufs, buf, group=group)
    return torch.cat([g.narrow(dim, 0, b - a) for g, (a, b) in zip(bufs, shards)], dim=dim)


def sharded_fwd(q, k, v, rand_attn, seq_mask=None, *, block: int = 64, r: int = 3, group=None, gather: bool = True,
                compute=None):
    """Head-sharded forward over a torch.distributed process group.

    Every rank passes the full-shape inputs it has (only its own heads are
    read): rank i of the group computes heads head_shard(H, world, i) of every
    sequence -- rand_attn is per head, so each rank takes its rows of it --
    and, with gather=True, the outputs are all-gathered along the head axis
    (NCCL over NVLink on GPUs). Heads are independent: the gather is the only
    exchange. Returns the full [B, H, L, d] output (gather=True) or this
    rank's [B, hi-lo, L, d] slice. Without an initialised process group the
    call computes every head itself.

    compute(q, k, v, rand_attn, seq_mask, block, r) defaults to the CUDA
    forward (bigbird_attn_fwd through the package's fwd()).
    """
    compute = compute or _default_compute()
    world, rank, dist_on = _group_info(group)
    B, H, L, d = q.shape
    if H < world:
        raise ValueError(f"{H} heads cannot be split over {world} ranks")
    lo, hi = head_shard(H, world, rank)
    sl = slice(lo, hi)
    part = compute(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(),
                   None if rand_attn is None else rand_attn[sl].contiguous(), seq_mask, block, r)
    if not gather or not dist_on:
        return part
    return _all_gather_along(part, 1, [head_shard(H, world, i) for i in range(world)], group)


def batch_sharded_fwd(q, k, v, rand_attn, seq_mask=None, *, block: int = 64, r: int = 3, group=None,
                      gather: bool = True, compute=None):
    """Batch-sharded forward over a torch.distributed process group: rank i
    computes sequences batch_shard(B, world, i) (every head, the shared
    rand_attn) and, with gather=True, the outputs are all-gathered along the
    batch axis. Returns [B, H, L, d] (gather=True) or this rank's
    [hi-lo, H, L, d] slice. compute as in sharded_fwd."""
    compute = compute or _default_compute()
    world, rank, dist_on = _group_info(group)
    B = q.shape[0]
    if B < world:
        raise ValueError(f"{B} sequences cannot be split over {world} ranks")
    lo, hi = batch_shard(B, world, rank)
    sm = None if seq_mask is None else seq_mask[lo:hi].contiguous()
    part = compute(q[lo:hi].contiguous(), k[lo:hi].contiguous(), v[lo:hi].contiguous(), rand_attn, sm, block, r)
    if not gather or not dist_on:
        return part
    return _all_gather_along(part, 0, [batch_shard(B, world, i) for i in range(world)], group)
