"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test names the plausible oracle mistake it would catch. None of these
tests touches the CUDA path.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_attention_b200.workloads import WORKLOADS, make_inputs, mask_from_lengths

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_qkv(B, H, L, d, seed, scale=1.0):
    g = np.random.default_rng(seed)
    mk = lambda: (g.standard_normal((B, H, L, d)) * scale)
    return mk(), mk(), mk()


def _sdpa_f64(q, k, v, seq_mask):
    """Full softmax attention from torch's library routine, fp64, key bias -10000."""
    q, k, v = (torch.from_numpy(np.asarray(x, np.float64)) for x in (q, k, v))
    B, H, L, d = q.shape
    if seq_mask is None:
        bias = torch.zeros(B, 1, 1, L, dtype=torch.float64)
    else:
        m = torch.as_tensor(np.asarray(seq_mask)).bool()
        bias = torch.where(m, 0.0, -10000.0).to(torch.float64).view(B, 1, 1, L)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=bias).numpy()


# ---------------------------------------------------------------- page values

def test_page_fallback_threshold():
    """704 = (5 + 2*3) * 64: the printed fallback length (catches an off-by-one
    in the fallback rule or a wrong count of minimum blocks)."""
    g = json.load(open(os.path.join(GOLDEN, "page_constants.json")))["fallback_threshold_tokens"]
    bs, r, thr = g["block_size"], g["num_random_blocks"], g["value"]
    assert oracle.is_fallback(thr, bs, r)
    assert not oracle.is_fallback(thr + bs, bs, r)
    assert all(oracle.is_fallback(L, bs, r) for L in range(bs, thr + 1, bs))


def test_page_head_dim_defaults():
    g = json.load(open(os.path.join(GOLDEN, "page_constants.json")))
    assert g["tf_defaults"]["hidden_size"] // g["tf_defaults"]["num_attention_heads"] == 64
    assert g["hf_defaults"]["d_model"] // g["hf_defaults"]["encoder_attention_heads"] == 64
    assert oracle.BIAS_MASKED == g["masked_bias"]["value"]


def test_argument_rules():
    with pytest.raises(ValueError):
        oracle.check_shape(1000, 64, 3)  # not a multiple of the block
    with pytest.raises(ValueError):
        oracle.check_shape(1024, 64, 0)  # r = 0 unsupported
    assert oracle.check_shape(1024, 64, 3) == 16


# ---------------------------------------------------------------- generator

def test_splitmix64_published_vectors():
    """Catches a wrong constant, shift or counter step in the generator."""
    g = json.load(open(os.path.join(GOLDEN, "splitmix64_vectors.json")))["streams"]
    s0 = [oracle.splitmix64_output(g[0]["seed"], n + 1) for n in range(4)]
    assert [f"{x:016x}" for x in s0] == g[0]["outputs_hex"]
    s1 = [oracle.splitmix64_output(g[1]["seed"], n + 1) for n in range(5)]
    assert [str(x) for x in s1] == g[1]["outputs_dec"]


@pytest.mark.parametrize("L,r,last_idx", [(1024, 3, 0), (4096, 3, 0), (640, 1, 0), (4096, 3, 1024), (2048, 5, 0)])
def test_generator_rules(L, r, last_idx):
    """Range, distinctness and window exclusion of every row
    (catches a pool that includes the window, a global block or a repeat)."""
    H, bs = 3, 64
    nb = L // bs
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=77, last_idx=last_idx)
    assert ra.shape == (H, nb - 2, r) and ra.dtype == np.int32
    oracle.rand_attn_validate(ra, H, L, bs, r, last_idx=last_idx)
    for h in range(H):
        for i in range(1, nb - 1):
            row = ra[h, i - 1]
            assert len(set(row.tolist())) == r
            assert all(1 <= x <= nb - 2 and not (i - 1 <= x <= i + 1) for x in row)
            if last_idx:
                assert all((x + 1) * bs <= last_idx for x in row)
    # determinism, and distinct streams per head and per seed
    assert np.array_equal(ra, oracle.rand_attn_generate(H, L, bs, r, seed=77, last_idx=last_idx))
    assert not np.array_equal(ra, oracle.rand_attn_generate(H, L, bs, r, seed=78, last_idx=last_idx))
    if nb > 10:
        assert not np.array_equal(ra[0], ra[1])


def test_generator_infeasible():
    with pytest.raises(ValueError):
        oracle.rand_attn_generate(1, 7 * 64, 64, 3, seed=1)  # middle pool has nb-5 = 2 < 3
    with pytest.raises(ValueError):
        oracle.rand_attn_generate(1, 4096, 64, 3, seed=1, last_idx=256)


def test_generator_uniform():
    """chi-square of candidate frequencies and of the first slot against the
    exact uniform law of a random r-subset [TFG-BigBird, 随机块掩码是如何生成的:
    a random permutation of the pool]. Catches a biased bounded draw or an
    off-by-one in the Fisher-Yates range."""
    from scipy.stats import chi2
    L, bs, r, H = 16 * 64, 64, 3, 400
    nb = L // bs
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=2024)
    for i in (1, 5, nb - 2):
        pool = [j for j in range(1, nb - 1) if not (i - 1 <= j <= i + 1)]
        n = len(pool)
        rows = ra[:, i - 1, :]
        cnt = np.array([(rows == j).sum() for j in pool], dtype=float)
        exp = H * r / n
        stat = ((cnt - exp) ** 2 / exp).sum()
        assert chi2.sf(stat, n - 1) > 1e-4, (i, cnt)
        first = np.array([(rows[:, 0] == j).sum() for j in pool], dtype=float)
        exp1 = H / n
        stat1 = ((first - exp1) ** 2 / exp1).sum()
        assert chi2.sf(stat1, n - 1) > 1e-4, (i, first)


def test_validator_rejects():
    H, L, bs, r = 1, 1024, 64, 3
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=5)
    bad = ra.copy(); bad[0, 4, 0] = 5  # row i=5 window block
    with pytest.raises(ValueError):
        oracle.rand_attn_validate(bad, H, L, bs, r)
    bad = ra.copy(); bad[0, 4, 1] = bad[0, 4, 0]
    with pytest.raises(ValueError):
        oracle.rand_attn_validate(bad, H, L, bs, r)
    bad = ra.copy(); bad[0, 4, 0] = 0  # a global block
    with pytest.raises(ValueError):
        oracle.rand_attn_validate(bad, H, L, bs, r)


# ---------------------------------------------------------------- pattern

def test_block_mask_counts():
    """Rows 0, nb-1 see nb blocks; rows 1, nb-2 see 4+r; the others 5+r
    (catches a dropped global column, window term or random term)."""
    H, L, bs, r = 2, 4096, 64, 3
    nb = L // bs
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=9)
    for h in range(H):
        bm = oracle.block_mask(nb, r, ra[h], True)
        cnt = bm.sum(axis=1)
        assert cnt[0] == nb and cnt[nb - 1] == nb
        assert cnt[1] == 4 + r and cnt[nb - 2] == 4 + r
        assert (cnt[2:nb - 2] == 5 + r).all()
        assert bm[:, 0].all() and bm[:, nb - 1].all()
    assert oracle.keys_per_row(L, bs, r) == 622.0
    assert oracle.keys_per_row(1024, bs, r) == 568.0
    assert oracle.keys_per_row(L, bs, r, rand_attn=ra) == 622.0


def test_pattern_table_matches_rules():
    H, L, bs, r = 2, 1024, 64, 3
    nb = L // bs
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=3)
    pt = oracle.pattern_table(ra, H, L, bs, r)
    assert pt.shape == (H, nb - 2, 5 + r)
    for h in range(H):
        for i in range(1, nb - 1):
            want = sorted({0, nb - 1, i - 1, i, i + 1} | set(ra[h, i - 1].tolist()))
            got = [x for x in pt[h, i - 1].tolist() if x >= 0]
            assert got == want


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("L,pad", [(512, None), (704, [700]), (64 * 11, [300])])
def test_fallback_is_textbook_attention(L, pad):
    """nb <= 5 + 2r: the oracle equals torch's fp64 SDPA with the key bias
    (catches a wrong scale, a transposed operand or a sign error in the bias)."""
    B, H, d, bs, r = 1, 2, 32, 64, 3
    q, k, v = _rand_qkv(B, H, L, d, seed=L)
    sm = None if pad is None else mask_from_lengths(B, L, pad).numpy()
    got = oracle.attention(q, k, v, None, sm, bs, r)
    want = _sdpa_f64(q, k, v, sm)
    assert np.abs(got - want).max() < 1e-12


@pytest.mark.parametrize("pad", [None, [900]])
def test_brute_force_gather_all_rows(pad):
    """Dense-mask oracle vs per-query gather built straight from the rules,
    on every row of a 16-block sequence (catches any pattern mistake)."""
    B, H, L, d, bs, r = 1, 2, 1024, 16, 64, 3
    q, k, v = _rand_qkv(B, H, L, d, seed=11)
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=4)
    sm = None if pad is None else mask_from_lengths(B, L, pad).numpy()
    full = oracle.attention(q, k, v, ra, sm, bs, r)
    for h in range(H):
        rows = np.arange(L)
        bf = oracle.brute_force_rows(q, k, v, ra, sm, bs, r, 0, h, rows)
        assert np.abs(full[0, h] - bf).max() < 1e-12
        ar = oracle.attention_rows(q, k, v, ra, sm, bs, r, 0, h, rows[::7])
        assert np.abs(full[0, h, ::7] - ar).max() < 1e-13


def test_brute_force_sampled_base_shape():
    """The BigBird-base shape (L=4096, padding) on sampled rows."""
    w = WORKLOADS["bigbird_base_l4096"].with_(B=1, H=2)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
    rows = np.r_[0:3, 63:70, 128:131, 2000:2003, 4030:4096:9]
    for h in range(w.H):
        a = oracle.attention_rows(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r, 0, h, rows)
        b = oracle.brute_force_rows(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r, 0, h, rows)
        assert np.abs(a - b).max() < 1e-12


def test_rows_sum_to_one_and_q_zero_closed_form():
    """Q = 0: every attended valid key gets the same weight, so the output is
    the plain mean of v over the row's valid in-pattern keys (catches a bias
    sign error, a wrong row->rand_attn index, or weights that do not sum to 1)."""
    B, H, L, d, bs, r = 1, 1, 1024, 8, 64, 3
    nb = L // bs
    _, k, v = _rand_qkv(B, H, L, d, seed=5)
    q = np.zeros_like(k)
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=6)
    vl = 1000
    sm = mask_from_lengths(B, L, [vl]).numpy()
    out = oracle.attention(q, k, v, ra, sm, bs, r)
    for i in range(nb):
        if i in (0, nb - 1):
            blocks = range(nb)
        else:
            blocks = {0, nb - 1, i - 1, i, i + 1} | set(ra[0, i - 1].tolist())
        keys = [t for j in blocks for t in range(j * bs, (j + 1) * bs) if t < vl]
        want = v[0, 0, keys].mean(axis=0)
        assert np.abs(out[0, 0, i * bs:(i + 1) * bs] - want).max() < 1e-12
    # constant V => constant output (weights sum to one)
    vc = np.full_like(v, 0.375)
    qn, kn, _ = _rand_qkv(B, H, L, d, seed=8, scale=3.0)
    oc = oracle.attention(qn, kn, vc, ra, sm, bs, r)
    assert np.abs(oc - 0.375).max() < 1e-12


def test_all_keys_padded_is_shift_invariant():
    """A sequence whose keys are all padded adds the same -10000 to every
    score: the softmax is unchanged, so the result equals the unpadded one."""
    B, H, L, d, bs, r = 1, 1, 1024, 16, 64, 3
    q, k, v = _rand_qkv(B, H, L, d, seed=12)
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=1)
    sm0 = np.zeros((1, L), np.uint8)
    a = oracle.attention(q, k, v, ra, sm0, bs, r)
    b = oracle.attention(q, k, v, ra, None, bs, r)
    assert np.abs(a - b).max() < 1e-9


def test_padded_key_gets_zero_weight():
    """One padded key among valid ones contributes exp(-10000) = 0."""
    B, H, L, d, bs, r = 1, 1, 704, 16, 64, 3
    q, k, v = _rand_qkv(B, H, L, d, seed=13)
    sm = np.ones((1, L), np.uint8); sm[0, 5] = 0
    v2 = v.copy(); v2[0, 0, 5] = 1e6  # a huge value on the padded key changes nothing
    a = oracle.attention(q, k, v, None, sm, bs, r)
    b = oracle.attention(q, k, v2, None, sm, bs, r)
    assert np.abs(a - b).max() < 1e-12


def test_random_order_and_duplicates_are_set_semantics():
    """Permuting a row's random entries leaves the output unchanged; a random
    entry repeating a window or global block adds nothing (set semantics)."""
    B, H, L, d, bs, r = 1, 1, 1024, 16, 64, 3
    q, k, v = _rand_qkv(B, H, L, d, seed=14)
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=2)
    a = oracle.attention(q, k, v, ra, None, bs, r)
    b = oracle.attention(q, k, v, ra[:, :, ::-1].copy(), None, bs, r)
    assert np.abs(a - b).max() < 1e-13
    ra2 = ra.copy(); ra2[0, 4, 2] = 0  # row 5: replace one random block by global block 0
    c = oracle.attention(q, k, v, ra2, None, bs, r)
    ra3 = ra.copy(); ra3[0, 4, 2] = ra3[0, 4, 1]
    e = oracle.attention(q, k, v, ra3, None, bs, r)
    assert np.abs(c[0, 0, 5 * bs:6 * bs] - e[0, 0, 5 * bs:6 * bs]).max() < 1e-13
    bf = oracle.brute_force_rows(q, k, v, ra2, None, bs, r, 0, 0, np.arange(5 * bs, 6 * bs))
    assert np.abs(c[0, 0, 5 * bs:6 * bs] - bf).max() < 1e-12


def test_forced_sparse_full_coverage():
    """nb = 5 + r with the middle rows' random blocks = all remaining middle
    blocks: those rows cover every block and equal full attention."""
    B, H, d, bs, r = 1, 1, 16, 64, 3
    nb = 5 + r
    L = nb * bs
    q, k, v = _rand_qkv(B, H, L, d, seed=15)
    ra = oracle.rand_attn_generate(H, L, bs, r, seed=3)
    for i in range(2, nb - 2):
        rest = [j for j in range(1, nb - 1) if not (i - 1 <= j <= i + 1)]
        assert len(rest) == r
        ra[0, i - 1] = rest
    sp = oracle.attention(q, k, v, ra, None, bs, r, force_sparse=True)
    full = _sdpa_f64(q, k, v, None)
    assert np.abs(sp[0, 0, 2 * bs:(nb - 2) * bs] - full[0, 0, 2 * bs:(nb - 2) * bs]).max() < 1e-12
    # rows 1 and nb-2 miss exactly one block, so they must differ
    assert np.abs(sp[0, 0, bs:2 * bs] - full[0, 0, bs:2 * bs]).max() > 1e-6


def test_mask_prep_from_positions():
    """blocked/band/from/to masks against validity computed from token
    positions and valid lengths alone (catches a wrong window offset)."""
    B, L, bs = 3, 1024, 64
    nb = L // bs
    vl = [1024, 700, 130]
    sm = mask_from_lengths(B, L, vl).numpy()
    blocked, band, frm, to = oracle.mask_prep(sm, bs)
    assert blocked.shape == (B, nb, bs) and band.shape == (B, nb - 4, bs, 3 * bs)
    for b in range(B):
        ok = lambda t: int(t < vl[b])
        for j in range(nb):
            assert [int(x) for x in blocked[b, j]] == [ok(j * bs + t) for t in range(bs)]
        for i in range(2, nb - 2):
            for x in (0, 17, 63):
                for w in range(3):
                    for y in (0, 31, 63):
                        assert band[b, i - 2, x, w * bs + y] == ok(i * bs + x) * ok((i - 1 + w) * bs + y)
        assert [int(t) for t in frm[b]] == [ok(t) for t in range(L)]
        assert np.array_equal(frm, to)


def test_bf16_inputs_used_exactly():
    """Torch bf16 inputs enter at their exact values."""
    w = WORKLOADS["tiny_l1024"].with_(H=1)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
    a = oracle.attention(inp["q"], inp["k"], inp["v"], ra, None, w.block, w.r)
    b = oracle.attention(inp["q"].float().numpy(), inp["k"].float().numpy(),
                         inp["v"].float().numpy(), ra, None, w.block, w.r)
    assert np.array_equal(a, b)


def test_sparse_flops():
    assert oracle.sparse_flops(4, 12, 4096, 64, 64, 3) == 4.0 * 4 * 12 * 4096 * 622 * 64
    assert math.isclose(oracle.sparse_flops(4, 12, 4096, 64, 64, 3) / 1e9, 31.31, rel_tol=1e-3)


@pytest.mark.parametrize("L,d", [(1024, 64), (20 * 64, 32), (11 * 64, 16)])
def test_work_counts_match_the_attended_pairs(L, d):
    """The forward and backward work counts equal a count of the attended
    (query, key) pairs taken from the weight matrix itself: every attended
    pair has a nonzero weight (no padding here), every other pair weight 0.
    Per pair and head dimension the forward forms 2 products (q.k and p.v)
    and the backward 5 (q.k recomputed, dout.v, p.dout, ds.k, ds.q), each
    one multiply-add = 2 FLOP."""
    B, H, block, r = 1, 2, 64, 3
    q, k, _ = _rand_qkv(B, H, L, d, seed=41)
    nb = L // block
    ra = None if oracle.is_fallback(L, block, r) else oracle.rand_attn_generate(H, L, block, r, seed=42)
    p = oracle.attention_probs(q, k, ra, None, block, r)
    pairs = int(np.count_nonzero(p))
    assert pairs > 0 and (pairs < B * H * L * L or nb <= 5 + 2 * r)
    assert oracle.sparse_flops(B, H, L, d, block, r) == 4.0 * d * pairs
    assert oracle.backward_flops(B, H, L, d, block, r) == 10.0 * d * pairs


# --------------------------------------------------------------------------
# The C sparse brute-force reference (the timed CPU baseline) against the
# dense-mask oracle: both are fp64 statements of the same definition, one by
# per-row key gathering in C, the other by an [L, L] mask in NumPy.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", ["sparse_padded", "fallback", "forced_sparse", "set_semantics", "all_padded"])
def test_c_sparse_reference_matches_oracle(case):
    from oracle import sparse_ref
    from block_sparse_long_attention_b200.workloads import Workload

    force = False
    if case == "sparse_padded":
        w = Workload("c", 2, 3, 21 * 64, pad=("fixed", [1300, 900]), seed=41)
    elif case == "fallback":
        w = Workload("c", 1, 2, 704, pad=("fixed", [500]), seed=42)
    elif case == "forced_sparse":
        w = Workload("c", 1, 2, 9 * 64, seed=43)
        force = True
    elif case == "set_semantics":
        w = Workload("c", 1, 2, 16 * 64, seed=44)
    else:
        w = Workload("c", 1, 1, 12 * 64, pad=("fixed", [0]), seed=45)
    inp = make_inputs(w)
    nb = w.L // w.block
    sparse = force or nb > 5 + 2 * w.r
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=7) if sparse else None
    if case == "set_semantics":
        ra[0] = 0                   # all-zero adjacency (global block repeated)
        ra[1, 4, :] = 5             # window overlap, repeated
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r, force_sparse=force)
    got = sparse_ref.sparse_attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r,
                                      force_sparse=force, threads=2)
    assert np.abs(got - want).max() < 1e-12


def test_c_sparse_reference_rejects_bad_input():
    from oracle import sparse_ref

    q = torch.zeros(1, 1, 12 * 64, 64, dtype=torch.bfloat16)
    ra = np.zeros((1, 10, 3), dtype=np.int32)
    ra[0, 2, 1] = 99
    with pytest.raises(ValueError):
        sparse_ref.sparse_attention(q, q, q, ra, None, 64, 3)


# --------------------------------------------------------------------------
# Backward pass of the oracle: pinned by finite differences of the forward
# (an independent route to the same derivatives) and by exact identities.
# --------------------------------------------------------------------------

def _fd_case(L, pad, seed):
    rng = np.random.default_rng(seed)
    B, H, d = 1, 2, 64
    q = rng.standard_normal((B, H, L, d)) * 0.5
    k = rng.standard_normal((B, H, L, d)) * 0.5
    v = rng.standard_normal((B, H, L, d))
    do = rng.standard_normal((B, H, L, d))
    sm = None if pad is None else mask_from_lengths(B, L, [pad]).numpy()
    ra = None if oracle.is_fallback(L, 64, 3) else oracle.rand_attn_generate(H, L, 64, 3, seed=seed)
    return q, k, v, do, sm, ra


@pytest.mark.parametrize("L,pad", [(12 * 64, 700), (704, None)], ids=["sparse_padded", "fallback"])
def test_backward_matches_finite_differences(L, pad):
    q, k, v, do, sm, ra = _fd_case(L, pad, seed=5)
    dq, dk, dv = oracle.attention_backward(q, k, v, ra, sm, 64, 3, do)

    def loss(qq, kk, vv):
        return float((oracle.attention(qq, kk, vv, ra, sm, 64, 3) * do).sum())

    rng = np.random.default_rng(11)
    eps = 1e-5
    for name, g in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(8):
            idx = (0, int(rng.integers(2)), int(rng.integers(L)), int(rng.integers(64)))
            plus = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            minus = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            plus[name][idx] += eps
            minus[name][idx] -= eps
            fd = (loss(plus["q"], plus["k"], plus["v"]) - loss(minus["q"], minus["k"], minus["v"])) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * (1 + abs(fd)), (name, idx, fd, g[idx])


def test_backward_identities():
    """Exact for any input: the rows of ds sum to zero, so sum_k dk = 0; the
    rows of p sum to one, so sum_k dv = sum_q dout. A padded key (-10000)
    receives nothing."""
    q, k, v, do, sm, ra = _fd_case(16 * 64, 900, seed=8)
    dq, dk, dv = oracle.attention_backward(q, k, v, ra, sm, 64, 3, do)
    assert np.abs(dk.sum(axis=2)).max() < 1e-10
    assert np.abs(dv.sum(axis=2) - do.sum(axis=2)).max() < 1e-10
    assert np.abs(dk[:, :, 900:]).max() == 0.0 and np.abs(dv[:, :, 900:]).max() == 0.0
    # identical keys: every score of a row is equal, so q gets no gradient
    kc = np.broadcast_to(k[:, :, :1], k.shape).copy()
    dq2, _, _ = oracle.attention_backward(q, kc, v, ra, None, 64, 3, do)
    assert np.abs(dq2).max() < 1e-12


def test_lse_is_the_softmax_normaliser():
    q, k, v, do, sm, ra = _fd_case(12 * 64, 600, seed=9)
    lse = oracle.attention_lse(q, k, ra, sm, 64, 3)
    # with v = one-hot of key t, the output is p[:, t] = exp(s[:, t] - lse)
    L = q.shape[2]
    t = 5
    e = np.zeros_like(v)
    e[..., t, 0] = 1.0
    p_t = oracle.attention(q, k, e, ra, sm, 64, 3)[..., 0]
    s_t = (q @ k[:, :, t:t + 1].transpose(0, 1, 3, 2))[..., 0] / 8.0   # key t is in block 0 (a global block)
    assert np.abs(p_t - np.exp(s_t - lse)).max() < 1e-12


# --------------------------------------------------------------------------
# Attention probabilities of the oracle: pinned through attention() itself
# (an identity value matrix turns its output into the weights) and through
# the closed form exp(s - lse).
# --------------------------------------------------------------------------

_PROBS_CASES = [(12 * 64, 700, False), (704, 600, False), (8 * 64, 450, True)]


@pytest.mark.parametrize("L,pad,force", _PROBS_CASES, ids=["sparse_padded", "fallback", "forced_sparse"])
def test_probs_are_attention_of_identity_values(L, pad, force):
    """With V = I (value of key k = the k-th unit vector) the output row q is
    the weight vector of row q. Catches a probability matrix whose support,
    scaling or normalisation differs from the (separately pinned) forward."""
    rng = np.random.default_rng(21)
    B, H, d, r = 1, 2, 64, 3
    q = rng.standard_normal((B, H, L, d)) * 0.6
    k = rng.standard_normal((B, H, L, d)) * 0.6
    sm = mask_from_lengths(B, L, [pad]).numpy()
    nb = L // 64
    if force:   # nb = 5 + r: the random blocks are the rest of the middle rows
        ra = np.zeros((H, nb - 2, r), dtype=np.int32)
        for h in range(H):
            for i in range(1, nb - 1):
                rest = [j for j in range(1, nb - 1) if abs(j - i) > 1]
                ra[h, i - 1, :len(rest)] = rest[:r]
                ra[h, i - 1, len(rest):] = rest[0]
    else:
        ra = None if oracle.is_fallback(L, 64, r) else oracle.rand_attn_generate(H, L, 64, r, seed=3)
    # V = I, 64 columns at a time (attention() takes values of the head width)
    eye = np.eye(L)
    want = np.concatenate([oracle.attention(q, k, np.broadcast_to(eye[:, c:c + d], (B, H, L, d)), ra, sm, 64, r,
                                            force_sparse=force) for c in range(0, L, d)], axis=3)
    got = oracle.attention_probs(q, k, ra, sm, 64, r, force_sparse=force)
    assert np.abs(got - want).max() < 1e-12
    assert np.abs(got.sum(axis=3) - 1.0).max() < 1e-12
    rows = [0, 63, 64, 200, L - 65, L - 1]
    assert np.array_equal(oracle.attention_probs_rows(q, k, ra, sm, 64, r, 0, 1, rows, force_sparse=force),
                          got[0, 1, rows])


def test_probs_closed_form_and_support():
    """probs = exp(s - lse) on the pattern, exactly 0 off it and on padded keys
    (for rows with a valid key). Catches a wrong score scale, a bias applied to
    the wrong side, or weight leaking outside the pattern."""
    rng = np.random.default_rng(22)
    B, H, L, d, r = 2, 2, 16 * 64, 64, 3
    q = rng.standard_normal((B, H, L, d)) * 0.5
    k = rng.standard_normal((B, H, L, d)) * 0.5
    sm = mask_from_lengths(B, L, [1000, 700]).numpy()
    ra = oracle.rand_attn_generate(H, L, 64, r, seed=5)
    p = oracle.attention_probs(q, k, ra, sm, 64, r)
    lse = oracle.attention_lse(q, k, ra, sm, 64, r)
    nb = L // 64
    for b in range(B):
        for h in range(H):
            s = q[b, h] @ k[b, h].T / 8.0 + np.where(sm[b].astype(bool), 0.0, -10000.0)[None, :]
            for i in range(nb):
                # key blocks of query block i, listed from the rules as the pages state them
                if i in (0, nb - 1):
                    blocks = set(range(nb))
                else:
                    blocks = {0, nb - 1, i - 1, i, i + 1} | {int(x) for x in ra[h, i - 1]}
                keys = np.concatenate([np.arange(j * 64, j * 64 + 64) for j in sorted(blocks)])
                rows = slice(i * 64, i * 64 + 64)
                off = np.setdiff1d(np.arange(L), keys)
                assert np.all(p[b, h, rows][:, off] == 0.0)
                want = np.exp(s[rows][:, keys] - lse[b, h, rows][:, None])
                assert np.abs(p[b, h, rows][:, keys] - want).max() < 1e-13
            valid = int(sm[b].sum())
            assert np.all(p[b, h, :, valid:] == 0.0)
