"""Backward pass (bigbird_attn_fwd_train + bigbird_attn_bwd through the C ABI)
against the fp64 oracle.

The GPU recomputes p from its own forward's log-sum-exp and uses its own
forward output in D = rowsum(dout * out); the oracle uses exact values. The
bar is relative to the size of each gradient. The backward itself is fp32
arithmetic on bf16 inputs (sums of <= L products: ~1e-6 relative); the
forward's output carries the error of its fp16 P (~1e-4 of |out|), which
reaches ds through D and bounds dq and dk at ~1e-4 of their scale (measured
1.2e-4 at most); dv does not depend on D (measured 1e-6).
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
import block_sparse_long_attention_b200 as bb
from block_sparse_long_attention_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

# max |err| <= MAX_REL * max |ref|, mean |err| <= MEAN_REL * mean |ref|
MAX_REL, MEAN_REL = 1e-3, 2e-4
LSE_MAX_ABS = 1e-5
REPORT = os.environ.get("BB_TEST_REPORT")  # optional JSON-lines file for the measured errors


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_attention_b200 import build
    build.build()
    bb.device_status()
    yield


def _report(**kw):
    if not REPORT:
        return
    try:
        os.makedirs(os.path.dirname(REPORT) or ".", exist_ok=True)
        with open(REPORT, "a") as f:
            f.write(json.dumps(kw) + "\n")
    except OSError:
        pass


def _dout(w, seed=99):
    return torch.randn(w.B, w.H, w.L, 64, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)


def _run(inp, w, ra, dout, force_sparse=False):
    q, k, v = (inp[x].cuda() for x in "qkv")
    sm = None if inp["seq_mask"] is None else inp["seq_mask"].cuda()
    ra_d = None if ra is None else torch.from_numpy(np.ascontiguousarray(ra)).cuda()
    out, lse = bb.fwd_train(q, k, v, ra_d, sm, block=w.block, r=w.r, out_dtype=torch.float32,
                            force_sparse=force_sparse)
    dq, dk, dv = bb.bwd(q, k, v, out, dout.cuda(), lse, ra_d, sm, block=w.block, r=w.r, force_sparse=force_sparse)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    return [t.double().cpu().numpy() for t in (out, lse, dq, dk, dv)]


def _check_grad(name, got, want, what):
    err = np.abs(got - want)
    ref_max, ref_mean = float(np.abs(want).max()), float(np.abs(want).mean())
    _report(case=what, grad=name, max_err=float(err.max()), mean_err=float(err.mean()), ref_max=ref_max,
            ref_mean=ref_mean)
    assert np.isfinite(got).all(), (what, name)
    assert err.max() <= MAX_REL * ref_max, (what, name, float(err.max()), ref_max)
    assert err.mean() <= MEAN_REL * ref_mean, (what, name, float(err.mean()), ref_mean)


CASES = [
    WORKLOADS["tiny_l1024"],
    Workload("split3_padded", 2, 3, 24 * 64, pad=("fixed", [1000, 1536]), seed=8),
    Workload("pairs_odd_tail", 1, 2, 13 * 64, pad=("fixed", [800]), seed=7),
    Workload("fallback_704", 2, 2, 704, pad=("fixed", [700, 100]), seed=11),
    Workload("fallback_one_block", 1, 2, 64, seed=12),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_parity(w):
    inp = make_inputs(w)
    ra = None if oracle.is_fallback(w.L, w.block, w.r) else bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
    do = _dout(w)
    out, lse, dq, dk, dv = _run(inp, w, ra, do)
    want_lse = oracle.attention_lse(inp["q"], inp["k"], ra, inp["seq_mask"], w.block, w.r)
    _report(case=w.name, grad="lse", max_err=float(np.abs(lse - want_lse).max()))
    assert np.abs(lse - want_lse).max() <= LSE_MAX_ABS
    gq, gk, gv = oracle.attention_backward(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r, do)
    for name, got, want in (("dq", dq, gq), ("dk", dk, gk), ("dv", dv, gv)):
        _check_grad(name, got, want, w.name)


def test_backward_set_semantics():
    """Duplicate and window-overlapping random entries add nothing, as in the forward."""
    w = Workload("bwd_edge", 1, 2, 16 * 64, pad=("fixed", [900]), seed=17)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=4)
    ra[0] = 0
    ra[1, 5, :] = ra[1, 5, 0]
    ra[1, 9, 0] = 10
    do = _dout(w, 5)
    out, lse, dq, dk, dv = _run(inp, w, ra, do)
    gq, gk, gv = oracle.attention_backward(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r, do)
    for name, got, want in (("dq", dq, gq), ("dk", dk, gk), ("dv", dv, gv)):
        _check_grad(name, got, want, w.name)


def test_backward_full_size_head_and_identities():
    """The BigBird-base workload: one whole (b, h) head against the oracle, and
    on every head the identities sum_k dk = 0 and sum_k dv = sum_q dout."""
    w = WORKLOADS["bigbird_base_l4096"]
    inp = make_inputs(w)
    ra = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
    do = _dout(w, 7)
    out, lse, dq, dk, dv = _run(inp, w, ra, do)
    b, h = 1, 5
    sub = {x: inp[x][b:b + 1, h:h + 1] for x in "qkv"}
    gq, gk, gv = oracle.attention_backward(sub["q"], sub["k"], sub["v"], ra[h:h + 1], inp["seq_mask"][b:b + 1].numpy(),
                                           w.block, w.r, do[b:b + 1, h:h + 1])
    for name, got, want in (("dq", dq[b:b + 1, h:h + 1], gq), ("dk", dk[b:b + 1, h:h + 1], gk),
                            ("dv", dv[b:b + 1, h:h + 1], gv)):
        _check_grad(name, got, want, "base_head")
    dsum = do.double().numpy().sum(axis=2)
    scale_k = np.abs(dk).sum(axis=2).max()
    _report(case="base_identities", dk_sum=float(np.abs(dk.sum(axis=2)).max()), dk_scale=float(scale_k),
            dv_sum_err=float(np.abs(dv.sum(axis=2) - dsum).max()))
    assert np.abs(dk.sum(axis=2)).max() <= 2e-4 * scale_k
    assert np.abs(dv.sum(axis=2) - dsum).max() <= 2e-4 * np.abs(dsum).max()


def test_backward_deterministic_and_long_transposed_lists():
    """The gradients are the same bit for bit on a second run (no atomics),
    and a key block picked by every middle row's random entries (a transposed
    list longer than one chunk of the dk/dv kernel) is handled."""
    w = Workload("bwd_chunks", 1, 2, 64 * 64, pad=("fixed", [3900]), seed=21)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=6)
    nb = w.nb
    for h in range(w.H):  # every middle row outside block 5's window picks block 5 (set semantics elsewhere)
        for i in range(1, nb - 1):
            if abs(i - 5) > 1:
                ra[h, i - 1, 0] = 5
    do = _dout(w, 8)
    first = _run(inp, w, ra, do)
    again = _run(inp, w, ra, do)
    for a, b in zip(first[2:], again[2:]):
        assert np.array_equal(a, b)
    out, lse, dq, dk, dv = first
    gq, gk, gv = oracle.attention_backward(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r, do)
    for name, got, want in (("dq", dq, gq), ("dk", dk, gk), ("dv", dv, gv)):
        _check_grad(name, got, want, w.name)


OTHER_SIZES = [(128, 64), (64, 128), (128, 128)]  # (block, d)


def _run_bd(inp, w, ra, dout):
    q, k, v = (inp[x].cuda() for x in "qkv")
    sm = None if inp["seq_mask"] is None else inp["seq_mask"].cuda()
    ra_d = None if ra is None else torch.from_numpy(np.ascontiguousarray(ra)).cuda()
    out, lse = bb.fwd_train(q, k, v, ra_d, sm, block=w.block, r=w.r, out_dtype=torch.float32)
    grads = bb.bwd(q, k, v, out, dout.cuda(), lse, ra_d, sm, block=w.block, r=w.r)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    return [t.double().cpu().numpy() for t in grads]


@pytest.mark.parametrize("block,d", OTHER_SIZES, ids=[f"b{b}_d{d}" for b, d in OTHER_SIZES])
def test_backward_other_sizes(block, d):
    """Blocks of 128 (two 64-token tiles: the dk/dv kernel's units are single
    key blocks) and d = 128 (two 64-column chunks; one CTA per SM): a padded
    sparse case with split global rows and a full-attention case, against
    the oracle, and a bit-exact second run."""
    cases = [
        Workload(f"bwd_sparse_b{block}_d{d}", 2, 2, 14 * block, d=d, block=block, value_scale=1.0,
                 pad=("fixed", [14 * block - 70, 9 * block + 5]), seed=71 + d + block),
        Workload(f"bwd_fallback_b{block}_d{d}", 1, 2, 8 * block, d=d, block=block, pad=("fixed", [8 * block - 3]),
                 seed=72 + d + block),
    ]
    for w in cases:
        inp = make_inputs(w)
        ra = None if oracle.is_fallback(w.L, w.block, w.r) else bb.rand_attn_generate(w.H, w.L, w.block, w.r,
                                                                                      seed=w.seed)
        do = torch.randn(w.B, w.H, w.L, d, generator=torch.Generator().manual_seed(w.seed)).to(torch.bfloat16)
        dq, dk, dv = _run_bd(inp, w, ra, do)
        again = _run_bd(inp, w, ra, do)
        for a, b in zip((dq, dk, dv), again):
            assert np.array_equal(a, b)
        gq, gk, gv = oracle.attention_backward(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r, do)
        for name, got, want in (("dq", dq, gq), ("dk", dk, gk), ("dv", dv, gv)):
            _check_grad(name, got, want, w.name)


@pytest.mark.parametrize("block", [64, 128], ids=["b64", "b128"])
def test_forward_and_backward_at_max_r(block):
    """r = 16, the largest supported: a pair of 64-token query blocks has 38
    candidate key blocks (window, global, 32 random), and a key block of the
    dk/dv kernel is picked by many query blocks. Entries 10..15 of every row
    repeat blocks listed before them (the row's first entry, a global block,
    its own window block, the previous row's entry), some with the other
    half of a pair, which set semantics merges [TFG-BigBird, section
    "随机块掩码是如何生成的"]. Forward output and lse, and dq, dk, dv against
    the oracle; the gradients the same on a second run."""
    nb = 40
    w = Workload(f"max_r_b{block}", 1, 2, nb * block, block=block, r=16, pad=("fixed", [nb * block - 150]),
                 seed=91 + block)
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
    do = _dout(w, 13)
    out, lse, dq, dk, dv = _run(inp, w, ra, do)
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r)
    ferr = np.abs(out - want)
    _report(case=w.name, grad="out", max_err=float(ferr.max()), mean_err=float(ferr.mean()))
    assert ferr.max() <= 1e-2 and ferr.mean() <= 1e-3, (float(ferr.max()), float(ferr.mean()))
    want_lse = oracle.attention_lse(inp["q"], inp["k"], ra, inp["seq_mask"], w.block, w.r)
    assert np.abs(lse - want_lse).max() <= LSE_MAX_ABS
    again = _run(inp, w, ra, do)
    for a, b in zip((dq, dk, dv), again[2:]):
        assert np.array_equal(a, b)
    gq, gk, gv = oracle.attention_backward(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r, do)
    for name, got, want_g in (("dq", dq, gq), ("dk", dk, gk), ("dv", dv, gv)):
        _check_grad(name, got, want_g, w.name)
