"""Multi-rank host logic on CPU (gloo, world size 2): each rank computes its
shard of a global batch independently; the gathered result equals the
single-process one, with no data-path exchange beyond the final gather."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_attention_b200.sharding import batch_shard


def test_batch_shard_covers_exactly():
    for gb in range(0, 13):
        for world in range(1, 6):
            owned = []
            for r in range(world):
                lo, hi = batch_shard(gb, world, r)
                owned.extend(range(lo, hi))
                assert hi - lo in (gb // world, gb // world + 1)
            assert owned == list(range(gb))
    with pytest.raises(ValueError):
        batch_shard(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _oracle_compute(q, k, v, ra_, sm, block, r):
    import oracle
    return torch.from_numpy(oracle.attention(q, k, v, None if ra_ is None else np.asarray(ra_),
                                             None if sm is None else np.asarray(sm), block, r))


def _worker(rank, world, port, result_path):
    """Each rank runs the product's batch-sharded forward (its slice of the
    sequences, then the all-gather along the batch axis) with the oracle as
    the per-rank compute (no GPU here)."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import oracle
    from block_sparse_long_attention_b200.sharding import batch_sharded_fwd
    from block_sparse_long_attention_b200.workloads import Workload, make_inputs
    w = Workload("dist", 3, 2, 14 * 64, pad=("fixed", [896, 500, 700]), seed=31)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
    full = batch_sharded_fwd(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], block=w.block, r=w.r,
                             compute=_oracle_compute)
    mine = batch_sharded_fwd(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], block=w.block, r=w.r,
                             gather=False, compute=_oracle_compute)
    lo, hi = batch_shard(w.B, world, rank)
    assert mine.shape[0] == hi - lo
    if rank == 0:
        ref = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"].numpy(), w.block, w.r)
        np.save(result_path, np.array([np.abs(full.numpy() - ref).max(), float(full.shape[0])]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_equal_single_process(tmp_path):
    path = str(tmp_path / "res.npy")
    mp.start_processes(_worker, args=(2, _free_port(), path), nprocs=2, join=True, start_method="spawn")
    err, nseq = np.load(path)
    assert err == 0.0 and nseq == 3


def _head_worker(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import oracle
    from block_sparse_long_attention_b200.sharding import sharded_fwd
    from block_sparse_long_attention_b200.workloads import Workload, make_inputs
    w = Workload("heads", 2, 5, 14 * 64, pad=("fixed", [896, 600]), seed=33)   # 5 heads over 2 ranks: 3 + 2
    inp = make_inputs(w)
    ra = torch.from_numpy(oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed))

    full = sharded_fwd(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], block=w.block, r=w.r,
                       compute=_oracle_compute)
    if rank == 0:
        ref = oracle.attention(inp["q"], inp["k"], inp["v"], ra.numpy(), inp["seq_mask"].numpy(), w.block, w.r)
        np.save(result_path, np.array([np.abs(full.numpy() - ref).max(), float(full.shape[1])]))
    dist.barrier()
    dist.destroy_process_group()


def test_head_sharded_forward_two_gloo_ranks(tmp_path):
    """sharded_fwd: each rank computes its heads (with its rows of rand_attn),
    the all-gather along the head axis reproduces the single-process output."""
    path = str(tmp_path / "heads.npy")
    mp.start_processes(_head_worker, args=(2, _free_port(), path), nprocs=2, join=True, start_method="spawn")
    err, nheads = np.load(path)
    assert err == 0.0 and nheads == 5


def test_head_shard_covers_exactly():
    from block_sparse_long_attention_b200.sharding import head_shard
    for H in range(1, 17):
        for world in range(1, 9):
            owned = [h for r in range(world) for h in range(*head_shard(H, world, r))]
            assert owned == list(range(H))
