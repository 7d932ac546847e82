"""bigbird_attn_fwd_host (host buffers, copies pipelined with compute one
sequence at a time) against bigbird_attn_fwd_ex on device buffers: the same
kernels on the same per-sequence units, so the outputs are equal bit for bit."""

import numpy as np
import pytest
import torch

import block_sparse_long_attention_b200 as bb
from block_sparse_long_attention_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_attention_b200 import build
    build.build()
    bb.device_status()
    yield


CASES = [
    (Workload("host_sparse", 3, 2, 20 * 64, pad=("fixed", [1100, 1280, 700]), seed=41), torch.bfloat16),
    (Workload("host_sparse_f32", 5, 3, 16 * 64, pad=("fixed", [900, 1024, 64, 1000, 333]), seed=42), torch.float32),
    (Workload("host_fallback", 2, 2, 704, pad=("fixed", [700, 300]), seed=43), torch.bfloat16),
    (Workload("host_block128_d128", 2, 2, 16 * 128, d=128, block=128, pad=("fixed", [2000, 1500]), seed=44),
     torch.float32),
]


@pytest.mark.parametrize("w,out_dtype", CASES, ids=[c[0].name for c in CASES])
def test_host_buffers_equal_device_call(w, out_dtype):
    inp = make_inputs(w)
    sparse = not bb.is_fallback(w.L, w.block, w.r)
    ra = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed) if sparse else None
    q, k, v = (inp[x].cuda() for x in "qkv")
    sm = inp["seq_mask"].cuda()
    want = bb.fwd(q, k, v, None if ra is None else torch.from_numpy(ra).cuda(), sm, block=w.block, r=w.r,
                  out_dtype=out_dtype)
    pin = {x: inp[x].contiguous().pin_memory() for x in "qkv"}
    out = torch.empty(q.shape, dtype=out_dtype).pin_memory()
    scratch = torch.empty(bb.fwd_host_scratch_bytes(w.B, w.H, w.L, w.d, w.block, w.r), dtype=torch.uint8,
                          device="cuda")
    for _ in range(2):  # the scratch is reused without clearing
        out.zero_()
        bb.fwd_host(pin["q"], pin["k"], pin["v"], ra, inp["seq_mask"].contiguous().pin_memory(), out,
                    block=w.block, r=w.r, scratch=scratch)
        torch.cuda.current_stream().synchronize()
        assert bb.device_status() == 0
        assert torch.equal(out, want.cpu())
