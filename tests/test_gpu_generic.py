"""The forward at the sizes other than block = d = 64, through the C ABI
against the fp64 oracle: blocks of 64 or 128 at d 64 or 128 on the
tensor-core kernel (a block of 128 is two 64-token tiles, d 128 two 64-column
chunks), block 32 on the CUDA-core kernel.

Bars: bf16 output max |err| <= 1e-2, mean <= 1e-3 (the forward's bar) for
both kernels. fp32 output: tensor-core sizes at the same bar (fp16 P, as at
block 64); CUDA-core sizes max |err| <= 1e-4, derived from the arithmetic:
fp32 dot products and sums over at most L keys (~1e-6 relative), accurate
exp2f, and one fp32 rescale per 32-key chunk (<= ~60 per row: ~4e-6
relative), on outputs of magnitude <~ 4. lse (fwd_train) <= 1e-5 absolute.
"""

import numpy as np
import pytest
import torch

import oracle
import block_sparse_long_attention_b200 as bb
from block_sparse_long_attention_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

SIZES = [(32, 64), (128, 64), (32, 128), (64, 128), (128, 128)]  # (block, d)
TENSOR_CORE = {(128, 64), (64, 128), (128, 128)}  # sizes the tensor-core kernel takes (besides block = d = 64)


def _check_f32(block, d, err, name):
    """fp32-output bar of the kernel that runs (block, d)."""
    if (block, d) in TENSOR_CORE:
        assert err.max() <= 1e-2 and err.mean() <= 1e-3, (name, float(err.max()), float(err.mean()))
    else:
        assert err.max() <= 1e-4, (name, float(err.max()))


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_attention_b200 import build
    build.build()
    bb.device_status()
    yield


def _ra(w, seed=None):
    if oracle.is_fallback(w.L, w.block, w.r):
        return None
    ra = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed if seed is None else seed)
    assert np.array_equal(ra, oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed if seed is None else seed))
    return ra


def _run(w, inp, ra, out_dtype, train=False, force_sparse=False):
    q, k, v = (inp[x].cuda() for x in "qkv")
    sm = None if inp["seq_mask"] is None else inp["seq_mask"].cuda()
    ra_d = None if ra is None else torch.from_numpy(np.ascontiguousarray(ra)).cuda()
    if train:
        out, lse = bb.fwd_train(q, k, v, ra_d, sm, block=w.block, r=w.r, out_dtype=out_dtype,
                                force_sparse=force_sparse)
    else:
        out, lse = bb.fwd(q, k, v, ra_d, sm, block=w.block, r=w.r, out_dtype=out_dtype,
                          force_sparse=force_sparse), None
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    return out.float().cpu().numpy().astype(np.float64), None if lse is None else lse.double().cpu().numpy()


def _cases(block, d):
    s = 10 * block + d
    return [
        Workload(f"sparse_b{block}_d{d}", 2, 2, 14 * block, d=d, block=block,
                 value_scale=1.0, pad=("fixed", [14 * block - block - 5, 7 * block + 3]), seed=s),
        Workload(f"fallback_b{block}_d{d}", 1, 2, 8 * block, d=d, block=block, pad=("fixed", [8 * block - 9]),
                 seed=s + 1),
        Workload(f"one_block_b{block}_d{d}", 1, 1, block, d=d, block=block, seed=s + 2),
    ]


@pytest.mark.parametrize("block,d", SIZES, ids=[f"b{b}_d{d}" for b, d in SIZES])
def test_generic_all_rows(block, d):
    for w in _cases(block, d):
        inp = make_inputs(w)
        ra = _ra(w)
        want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r)
        got, lse = _run(w, inp, ra, torch.float32, train=True)
        _check_f32(block, d, np.abs(got - want), w.name)
        want_lse = oracle.attention_lse(inp["q"], inp["k"], ra, inp["seq_mask"], w.block, w.r)
        assert np.abs(lse - want_lse).max() <= 1e-5, (w.name, float(np.abs(lse - want_lse).max()))
        got16, _ = _run(w, inp, ra, torch.bfloat16)
        err16 = np.abs(got16 - want)
        assert err16.max() <= 1e-2 and err16.mean() <= 1e-3, (w.name, float(err16.max()), float(err16.mean()))


@pytest.mark.parametrize("block,d", [(128, 64), (128, 128), (32, 64)], ids=["b128_d64", "b128_d128", "b32_d64"])
def test_generic_l4096(block, d):
    """4096 tokens (32 to 128 blocks), padded, every row of two heads."""
    w = Workload(f"l4096_b{block}_d{d}", 1, 2, 4096, d=d, block=block, value_scale=1.0 / np.sqrt(d),
                 pad=("fixed", [3001]), seed=3 * block + d)
    inp = make_inputs(w)
    ra = _ra(w)
    got, _ = _run(w, inp, ra, torch.float32)
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r)
    _check_f32(block, d, np.abs(got - want), w.name)


def test_generic_set_semantics_forced_sparse_and_flags():
    w = Workload("edge_b32", 1, 2, 16 * 32, d=64, block=32, pad=("fixed", [400]), seed=77)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=4)
    ra[0] = 0
    ra[1, 5, :] = ra[1, 5, 0]
    ra[1, 9, 0] = 10
    got, _ = _run(w, inp, ra, torch.float32)
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r)
    assert np.abs(got - want).max() <= 1e-4
    # forced sparse at nb = 5 + r: the sparse definition everywhere, and rows
    # 2 .. nb-3 (window + globals + the r remaining blocks) see every block;
    # rows 1 and nb-2 hold 4 + r blocks, so they cannot
    w2 = Workload("forced_b128", 1, 1, 8 * 128, d=128, block=128, seed=78)
    inp2 = make_inputs(w2)
    nb = 8
    ra2 = np.zeros((1, nb - 2, 3), dtype=np.int32)
    for i in range(1, nb - 1):
        rest = [j for j in range(1, nb - 1) if abs(j - i) > 1]
        ra2[0, i - 1] = (rest + [rest[0]] * 3)[:3]
    got2, _ = _run(w2, inp2, ra2, torch.float32, force_sparse=True)
    want2 = oracle.attention(inp2["q"], inp2["k"], inp2["v"], ra2, None, 128, 3, force_sparse=True)
    _check_f32(128, 128, np.abs(got2 - want2), w2.name)
    full2 = oracle.attention(inp2["q"], inp2["k"], inp2["v"], None, None, 128, 3)  # full attention
    mid = slice(2 * 128, (nb - 2) * 128)
    _check_f32(128, 128, np.abs(got2[:, :, mid] - full2[:, :, mid]), w2.name + " middle rows")
    # an out-of-range entry is skipped and flagged
    q, k, v = (inp[x].cuda() for x in "qkv")
    bad = torch.from_numpy(np.ascontiguousarray(ra)).cuda()
    bad[0, 3, 1] = 999
    bb.device_status()
    bb.fwd(q, k, v, bad, inp["seq_mask"].cuda(), block=32, r=3)
    assert bb.device_status() & 1
    # deterministic
    a, _ = _run(w, inp, ra, torch.float32)
    assert np.array_equal(a, got)


def test_block128_tensor_core_edges():
    """Block 128 on the tensor-core kernel: duplicate and window-overlapping
    random entries (set semantics), forced sparse at nb = 5 + r, a flagged
    out-of-range entry, run-to-run equality; and a full-attention case too
    wide for one unit (r = 9, 22 blocks), which runs on the CUDA cores."""
    w = Workload("edge_b128", 1, 2, 14 * 128, d=64, block=128, value_scale=1.0, pad=("fixed", [1700]), seed=91)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=5)
    ra[0] = 0                       # every entry the global block 0
    ra[1, 5, :] = ra[1, 5, 0]       # one entry three times
    ra[1, 9, 0] = 10                # the window block of row 10
    got, _ = _run(w, inp, ra, torch.float32)
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r)
    _check_f32(128, 64, np.abs(got - want), w.name)
    again, _ = _run(w, inp, ra, torch.float32)
    assert np.array_equal(again, got)
    # forced sparse at nb = 5 + r
    w2 = Workload("forced_b128_d64", 1, 1, 8 * 128, d=64, block=128, seed=92)
    inp2 = make_inputs(w2)
    nb = 8
    ra2 = np.zeros((1, nb - 2, 3), dtype=np.int32)
    for i in range(1, nb - 1):
        rest = [j for j in range(1, nb - 1) if abs(j - i) > 1]
        ra2[0, i - 1] = (rest + [rest[0]] * 3)[:3]
    got2, _ = _run(w2, inp2, ra2, torch.float32, force_sparse=True)
    want2 = oracle.attention(inp2["q"], inp2["k"], inp2["v"], ra2, None, 128, 3, force_sparse=True)
    _check_f32(128, 64, np.abs(got2 - want2), w2.name)
    # out-of-range entry: skipped and flagged
    q, k, v = (inp[x].cuda() for x in "qkv")
    bad = torch.from_numpy(np.ascontiguousarray(ra)).cuda()
    bad[0, 3, 1] = 999
    bb.device_status()
    bb.fwd(q, k, v, bad, inp["seq_mask"].cuda(), block=128, r=3)
    torch.cuda.synchronize()
    assert bb.device_status() & 1
    # 22 blocks at r = 9: full attention over 44 tiles, wider than a unit's
    # list, so the CUDA-core kernel takes it (fp32 bar 1e-4)
    w3 = Workload("wide_fallback_b128", 1, 1, 22 * 128, d=64, block=128, r=9, pad=("fixed", [2500]), seed=93)
    assert bb.workspace_size(1, 1, w3.L, 64, 128, r=9) == 0
    inp3 = make_inputs(w3)
    got3, _ = _run(w3, inp3, None, torch.float32)
    want3 = oracle.attention(inp3["q"], inp3["k"], inp3["v"], None, inp3["seq_mask"], 128, 9)
    assert np.abs(got3 - want3).max() <= 1e-4


@pytest.mark.parametrize("block,d", [(64, 128), (128, 128)], ids=["b64_d128", "b128_d128"])
def test_d128_v_beyond_fp16_range(block, d):
    """d 128: one key block of V at magnitude 1e20 (fp16 cannot hold it, so
    the call is redone with bf16 P and V). Every output is finite; rows with
    no weight on that block meet the forward's bar; the others |err| <= 1e-2
    + 2^-7 * mass * 1e20 (weights rounded once to bf16, relative 2^-9; mass =
    the row's weight on the block, from the oracle with V = 1 there)."""
    w = Workload(f"bigv_b{block}_d{d}", 1, 2, 16 * block, d=d, block=block, value_scale=1.0,
                 pad=("fixed", [16 * block - 37]), seed=95)
    j = 4
    inp = make_inputs(w)
    ra = _ra(w)
    v = inp["v"].clone()
    big = torch.randn(w.B, w.H, block, d, generator=torch.Generator().manual_seed(6))
    v[:, :, j * block:(j + 1) * block] = (big / big.abs().max() * 1e20).to(torch.bfloat16)
    inp = dict(inp, v=v)
    got, _ = _run(w, inp, ra, torch.float32)
    assert np.isfinite(got).all()
    want = oracle.attention(inp["q"], inp["k"], v, ra, inp["seq_mask"], w.block, w.r)
    ind = np.zeros(v.shape, np.float64)
    ind[:, :, j * block:(j + 1) * block] = 1.0
    mass = oracle.attention(inp["q"], inp["k"], ind, ra, inp["seq_mask"], w.block, w.r)[..., :1]
    vmax = float(v[:, :, j * block:(j + 1) * block].float().abs().max())
    err = np.abs(got - want)
    off = (mass == 0)[..., 0]
    assert off.any() and (~off).any()
    assert err[off].max() <= 1e-2 and err[off].mean() <= 1e-3, float(err[off].max())
    assert (err <= 1e-2 + 2.0 ** -7 * mass * vmax).all()


@pytest.mark.parametrize("block,d", [(32, 64), (32, 128), (64, 128)], ids=["b32_d64", "b32_d128", "b64_d128"])
def test_max_r_with_duplicates(block, d):
    """r = 16, the largest supported, on the CUDA-core kernel (block 32) and
    the d = 128 tensor-core kernel: entries 10..15 of every row repeat blocks
    listed before them (the row's first entry, a global block, its window
    block, the previous row's entry), which set semantics lists once
    [TFG-BigBird, section "随机块掩码是如何生成的"]; output and lse against the
    oracle."""
    nb = 40
    w = Workload(f"max_r_b{block}_d{d}", 1, 2, nb * block, d=d, block=block, value_scale=1.0,
                 pad=("fixed", [nb * block - 3 * block // 2]), r=16, seed=31 + block + d)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=5)
    for x in range(nb - 2):  # row x: query block x + 1
        e = ra[1, x]
        e[10] = e[0]
        e[11] = 0
        e[12] = x
        e[13] = ra[1, x - 1, 3] if x >= 1 else nb - 1
        e[14] = nb - 1
        e[15] = e[14]
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r)
    got, lse = _run(w, inp, ra, torch.float32, train=True)
    _check_f32(block, d, np.abs(got - want), w.name)
    want_lse = oracle.attention_lse(inp["q"], inp["k"], ra, inp["seq_mask"], w.block, w.r)
    assert np.abs(lse - want_lse).max() <= 1e-5, (w.name, float(np.abs(lse - want_lse).max()))
