"""The sharded wrappers with their default compute, the CUDA forward through
the C ABI, on a one-rank NCCL process group on the single GPU: each wrapper
computes its shard and runs its all-gather, and the result matches the fp64
oracle head by head at the forward's bar (max 1e-2, mean 1e-3)."""

import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import block_sparse_long_attention_b200 as bb
from block_sparse_long_attention_b200.sharding import batch_sharded_fwd, sharded_fwd
from block_sparse_long_attention_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 1e-2, 1e-3


@pytest.fixture(scope="module")
def nccl_group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_attention_b200 import build
    build.build()
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("wrapper", [sharded_fwd, batch_sharded_fwd], ids=["heads", "batch"])
def test_wrapper_with_cuda_compute(nccl_group, wrapper):
    w = Workload("shard", 2, 5, 14 * 64, pad=("fixed", [896, 600]), seed=33)
    inp = make_inputs(w)
    ra = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
    assert np.array_equal(ra, oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed))
    q, k, v = (inp[x].cuda() for x in "qkv")
    out = wrapper(q, k, v, torch.from_numpy(ra).cuda(), inp["seq_mask"].cuda(), block=w.block, r=w.r)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    assert out.shape == q.shape and out.dtype == torch.bfloat16
    got = out.float().cpu().numpy()
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r)
    for b in range(w.B):
        for h in range(w.H):
            err = np.abs(got[b, h].astype(np.float64) - want[b, h])
            assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, float(err.max()))
