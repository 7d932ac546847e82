"""bigbird_attn_fwd_noalloc: the forward pass for callers that cannot allocate
device memory while they run (e.g. a serving loop that reserves all GPU memory
up front and must never reach the allocator, or its device-wide
synchronisation, inside a step). It uses a fixed scratch region held by the
library instead of a workspace. It runs the same kernels on the same inputs as
the allocating entry point, and those kernels are deterministic, so its output
must equal that entry point's bit for bit, call after call.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import block_sparse_long_attention_b200 as bb
from block_sparse_long_attention_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_attention_b200 import build
    build.build()
    bb.device_status()
    yield


def _noalloc(lib, q, k, v, ra, sm, out, w, out_dtype, flags=0):
    B, H, L, d = q.shape
    return lib.bigbird_attn_fwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), ra.data_ptr(), None if sm is None else sm.data_ptr(),
        out.data_ptr(), B, H, L, d, w.block, w.r, out_dtype, flags,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_allocating_entry_point_twice():
    # the BigBird-base workload splits its global rows, so it uses the scratch region
    w = WORKLOADS["bigbird_base_l4096"]
    assert bb.workspace_size(w.B, w.H, w.L) > 0
    lib = bb.lib()
    assert bb.workspace_size(w.B, w.H, w.L) <= lib.bigbird_attn_noalloc_scratch_bytes()
    inp = make_inputs(w)
    q, k, v = (inp[x].cuda() for x in "qkv")
    sm = inp["seq_mask"].cuda()
    ra = torch.from_numpy(bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)).cuda()
    ref = bb.fwd(q, k, v, ra, sm, out_dtype=torch.float32)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        st = _noalloc(lib, q, k, v, ra, sm, out, w, bb.BB_OUT_F32)
        assert st == bb.BB_OK, bb.status_string(st)
        torch.cuda.synchronize()
        assert bb.device_status() == 0
        assert torch.isfinite(out).all()
        # same kernels, same inputs: any scratch-offset slip would show here
        assert torch.equal(out, ref)


@pytest.mark.parametrize("block,d", [(128, 64), (64, 128), (128, 128)], ids=["b128_d64", "b64_d128", "b128_d128"])
def test_noalloc_other_tensor_core_sizes(block, d):
    """Blocks of 128 and d = 128 run the tensor-core kernel too: the scratch
    region holds their workspace (partials of 128 columns at d = 128)."""
    from block_sparse_long_attention_b200.workloads import Workload
    w = Workload(f"noalloc_b{block}_d{d}", 2, 3, 24 * block, d=d, block=block, value_scale=1.0,
                 pad=("fixed", [24 * block - 100, 12 * block]), seed=61)
    lib = bb.lib()
    need = bb.workspace_size(w.B, w.H, w.L, d, block)
    assert 256 < need <= lib.bigbird_attn_noalloc_scratch_bytes()
    inp = make_inputs(w)
    q, k, v = (inp[x].cuda() for x in "qkv")
    sm = inp["seq_mask"].cuda()
    ra = torch.from_numpy(bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)).cuda()
    ref = bb.fwd(q, k, v, ra, sm, block=block, out_dtype=torch.float32)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        st = _noalloc(lib, q, k, v, ra, sm, out, w, bb.BB_OUT_F32)
        assert st == bb.BB_OK, bb.status_string(st)
        torch.cuda.synchronize()
        assert bb.device_status() == 0
        assert torch.equal(out, ref)


def test_noalloc_rejects_what_does_not_fit():
    lib = bb.lib()
    w = WORKLOADS["tiny_l1024"]
    inp = make_inputs(w)
    q, k, v = (inp[x].cuda() for x in "qkv")
    ra = torch.from_numpy(bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)).cuda()
    out = torch.empty_like(q)
    # 64 heads of 32K tokens need far more scratch than the fixed region: rejected before any launch
    big = bb.workspace_size(1, 64, 32768)
    assert big > lib.bigbird_attn_noalloc_scratch_bytes()
    st = lib.bigbird_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), ra.data_ptr(), None, out.data_ptr(),
                                      1, 64, 32768, 64, 64, 3, bb.BB_OUT_BF16, 0,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bb.BB_ERR_UNSUPPORTED
    # debug checks allocate a host buffer: not offered here
    st = _noalloc(lib, q, k, v, ra, None, out, w, bb.BB_OUT_BF16, bb.BB_FLAG_DEBUG_CHECKS)
    assert st == bb.BB_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bb.device_status() == 0
