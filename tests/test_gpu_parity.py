"""CUDA path (through the C ABI) against the fp64 oracle.

Bar: max |out - oracle| <= 1e-2 and mean |out - oracle| <= 1e-3 on bf16
inputs (the oracle sees the same bf16 values). Index and mask work (the key
set of every row) is checked exactly with a probe. The extreme-length
workload is compared with fp32 output: with values N(0,1)*2 an output of
magnitude 4..8 has a bf16 half-ulp of 1.6e-2, above the max-abs bar, whatever
the kernel does.
"""

import numpy as np
import pytest
import torch

import oracle
import block_sparse_long_attention_b200 as bb
from block_sparse_long_attention_b200.workloads import WORKLOADS, Workload, make_inputs, mask_from_lengths

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 1e-2, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_attention_b200 import build
    build.build()
    bb.device_status()  # clear the error word
    yield


def _cuda_fwd(inp, w: Workload, ra, out_dtype=torch.float32, force_sparse=False, seq_mask="inp"):
    q, k, v = (inp[x].cuda() for x in "qkv")
    sm = inp["seq_mask"] if seq_mask == "inp" else seq_mask
    sm = None if sm is None else sm.cuda()
    ra_d = None if ra is None else torch.from_numpy(np.ascontiguousarray(ra)).cuda()
    out = bb.fwd(q, k, v, ra_d, sm, block=w.block, r=w.r, out_dtype=out_dtype, force_sparse=force_sparse)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    return out.float().cpu().numpy()


def _check(got, want, what=""):
    err = np.abs(got.astype(np.float64) - want)
    assert np.isfinite(got).all(), what
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (what, float(err.max()), float(err.mean()))
    return float(err.max()), float(err.mean())


def _rand_attn_pair(w: Workload, seed=None):
    """rand_attn as each side derives it from the seed; the two are bit-exact."""
    s = w.seed if seed is None else seed
    if oracle.is_fallback(w.L, w.block, w.r):
        return None, None
    ra_cuda = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=s)
    ra_orc = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=s)
    assert np.array_equal(ra_cuda, ra_orc)
    return ra_cuda, ra_orc


SMALL = [
    WORKLOADS["tiny_l1024"],
    Workload("pairs_odd_tail", 1, 2, 13 * 64, pad=("fixed", [800]), seed=7),
    Workload("split3_padded", 2, 3, 24 * 64, pad=("fixed", [1000, 1536]), seed=8),
    Workload("smallest_sparse", 1, 2, 12 * 64, seed=9),
    Workload("ragged_split", 1, 2, 21 * 64, pad=("fixed", [1300]), seed=10),
    Workload("fallback_704", 2, 2, 704, pad=("fixed", [700, 100]), seed=11),
    Workload("fallback_one_block", 1, 2, 64, seed=12),
    Workload("fallback_three_blocks", 2, 1, 192, pad=("fixed", [192, 65]), seed=13),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_parity_all_rows(w, out_dtype):
    inp = make_inputs(w)
    ra_c, ra_o = _rand_attn_pair(w)
    got = _cuda_fwd(inp, w, ra_c, out_dtype)
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra_o, inp["seq_mask"], w.block, w.r)
    _check(got, want, w.name)


def test_forced_sparse_coverage():
    """nb = 5 + r with the middle rows' random blocks = all remaining middle
    blocks: those rows equal full attention; all rows match the oracle."""
    w = Workload("forced", 1, 2, 8 * 64, seed=14)
    nb = w.nb
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=3)
    for h in range(w.H):
        for i in range(2, nb - 2):
            ra[h, i - 1] = [j for j in range(1, nb - 1) if not (i - 1 <= j <= i + 1)]
    got = _cuda_fwd(inp, w, ra, torch.float32, force_sparse=True)
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, None, w.block, w.r, force_sparse=True)
    _check(got, want, "forced")
    full = oracle.attention(inp["q"], inp["k"], inp["v"], None, None, w.block, w.r)
    _check(got[:, :, 2 * 64:(nb - 2) * 64], full[:, :, 2 * 64:(nb - 2) * 64], "coverage")


def _sample_rows(L, block, rng, n_rand=96):
    nb = L // block
    rows = set(range(0, block)) | set(range((nb - 1) * block, L))           # global rows
    rows |= set(range(block, 2 * block, 7)) | set(range((nb - 2) * block, (nb - 1) * block, 7))  # second rows
    for j in range(8, nb, 8):                                               # split boundaries
        rows |= {j * block - 1, j * block}
    rows |= set(rng.integers(0, L, size=n_rand).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("name,out_dtype", [
    ("bigbird_base_l4096", torch.bfloat16), ("bigbird_base_l4096", torch.float32),
    ("pegasus_large_l4096", torch.bfloat16), ("long_l16384", torch.float32),
    ("long_l16384", torch.bfloat16), ("extreme_l32768", torch.float32)])
def test_parity_full_size_sampled(name, out_dtype):
    """Full workload sizes in the bench's launch configuration; the oracle
    evaluates sampled rows (every global row included) of every (b, h)."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    ra_c, ra_o = _rand_attn_pair(w)
    got = _cuda_fwd(inp, w, ra_c, out_dtype)
    rng = np.random.default_rng(0)
    errs = []
    for b in range(w.B):
        for h in range(w.H):
            rows = _sample_rows(w.L, w.block, rng, n_rand=48)
            want = oracle.attention_rows(inp["q"], inp["k"], inp["v"], ra_o, inp["seq_mask"], w.block, w.r, b, h, rows)
            errs.append(np.abs(got[b, h, rows].astype(np.float64) - want))
    err = np.concatenate([e.ravel() for e in errs])
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (name, float(err.max()), float(err.mean()))


def test_parity_full_heads_base():
    """Two whole heads of the BigBird-base workload against the full oracle."""
    w = WORKLOADS["bigbird_base_l4096"]
    inp = make_inputs(w)
    ra_c, ra_o = _rand_attn_pair(w)
    got = _cuda_fwd(inp, w, ra_c, torch.bfloat16)
    for b, h in ((0, 0), (3, 11)):
        sub = {x: inp[x][b:b + 1, h:h + 1] for x in "qkv"}
        sm = None if inp["seq_mask"] is None else inp["seq_mask"][b:b + 1]
        want = oracle.attention(sub["q"], sub["k"], sub["v"], ra_o[h:h + 1], sm, w.block, w.r)
        _check(got[b:b + 1, h:h + 1], want, f"head {b},{h}")


def test_determinism_and_batch_slices():
    """Run-to-run and batch-slice results are bit-identical."""
    w = WORKLOADS["bigbird_base_l4096"]
    inp = make_inputs(w)
    ra, _ = _rand_attn_pair(w)
    a = _cuda_fwd(inp, w, ra, torch.bfloat16)
    b = _cuda_fwd(inp, w, ra, torch.bfloat16)
    assert np.array_equal(a, b)
    for bi in (0, 2):
        sl = {x: inp[x][bi:bi + 1].contiguous() for x in "qkv"}
        sl["seq_mask"] = inp["seq_mask"][bi:bi + 1].contiguous()
        c = _cuda_fwd(sl, w.with_(B=1), ra, torch.bfloat16)
        assert np.array_equal(a[bi:bi + 1], c)


@pytest.mark.parametrize("L,bs,r,plant", [(4096, 64, 3, False), (4096, 64, 16, True), (8192, 128, 16, True)],
                         ids=["block64_r3", "block64_r16_dups", "block128_r16_dups"])
def test_key_set_probe_exact(L, bs, r, plant):
    """Q = 0 and V one-hot by key block (d = nb = 64): every row's output is the
    fraction of its valid keys in each block, so the per-block key counts of
    every row are recovered exactly from the fp32 output. With r = 16 a pair
    of query blocks has 38 candidate key blocks (window, global, 32 random),
    more than one per lane of the warp that builds the list; the planted
    entries repeat blocks listed earlier (the row's own first entry, a global
    block, a window block, the previous row's entry), some of them with
    another half mask, which set semantics merges [TFG-BigBird, section
    "随机块掩码是如何生成的"]."""
    B, H = 2, 3
    nb = L // bs
    assert nb == 64
    vl = [L, L * 5 // 8]
    sm = mask_from_lengths(B, L, vl)
    q = torch.zeros(B, H, L, 64, dtype=torch.bfloat16)
    k = torch.randn(B, H, L, 64, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    v = torch.zeros(B, H, L, 64, dtype=torch.bfloat16)
    for j in range(nb):
        v[:, :, j * bs:(j + 1) * bs, j] = 1.0
    ra = bb.rand_attn_generate(H, L, bs, r, seed=21)
    if plant:
        for x in range(nb - 2):  # row x: query block x + 1
            e = ra[1, x]
            e[10] = e[0]
            e[11] = 0
            e[12] = x
            e[13] = ra[1, x - 1, 3] if x >= 1 else nb - 1
            e[14] = nb - 1
            e[15] = e[14]
    w = Workload("probe", B, H, L, block=bs, r=r, seed=0)
    got = _cuda_fwd({"q": q, "k": k, "v": v, "seq_mask": sm}, w, ra, torch.float32)
    for b in range(B):
        valid = np.arange(L) < vl[b]
        per_block_valid = valid.reshape(nb, bs).sum(axis=1)
        for h in range(H):
            bm = oracle.block_mask(nb, r, ra[h], True)
            counts = bm * per_block_valid[None, :]          # [q-block, key block]
            n_tot = counts.sum(axis=1)
            rec = got[b, h].reshape(nb, bs, 64) * n_tot[:, None, None]
            assert np.abs(rec - counts[:, None, :]).max() < 1e-3, (b, h)


def test_set_semantics_and_all_padded():
    """Duplicate / global-block random entries (e.g. an all-zero adjacency)
    and a sequence with every key padded match the oracle's definition."""
    w = Workload("edge", 2, 2, 20 * 64, pad=("fixed", [1280, 0]), seed=17)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=4)
    ra[0] = 0                        # eval-mode style zero adjacency for head 0
    ra[1, 5, :] = ra[1, 5, 0]        # repeated entry
    ra[1, 9, 0] = 10                 # a window block of row 10
    got = _cuda_fwd(inp, w, ra, torch.float32)
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra, inp["seq_mask"], w.block, w.r)
    _check(got, want, "edge")


def test_max_growth_inside_and_across_blocks():
    """Scores that rise by about 16 (log2 units) from each 16-key piece of a
    block to the next and by about 17 from block to block: the lazy rescale
    (threshold 14) fires inside every block, after P of earlier pieces is
    written, and between blocks, after earlier P.V is in O; both repairs must
    give the oracle's softmax."""
    B, H, L = 1, 2, 12 * 64
    j = torch.arange(L, dtype=torch.float32)
    a = 0.35 * (j % 64) + 6.0 * (j // 64)     # score = q.k / 8 = 2a
    q = torch.full((B, H, L, 64), 0.25).to(torch.bfloat16)
    k = (a[:, None] * torch.ones(64)).expand(B, H, L, 64).contiguous().to(torch.bfloat16)
    v = torch.randn(B, H, L, 64, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    w = Workload("growth", B, H, L, seed=0)
    ra, ra_o = _rand_attn_pair(w, seed=31)
    got = _cuda_fwd({"q": q, "k": k, "v": v, "seq_mask": None}, w, ra, torch.float32)
    want = oracle.attention(q, k, v, ra_o, None, w.block, w.r)
    _check(got, want, "growth")


@pytest.mark.parametrize("vmax", [65280.0, 1.0e5, 1.0e20], ids=["fp16_edge", "1e5", "1e20"])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_v_beyond_fp16_range(vmax, out_dtype):
    """One key block of V scaled so its largest magnitude is vmax: 65280 is the
    largest bf16 value fp16 still holds, 1e5 and 1e20 are not representable in
    fp16 (the call is then done again with bf16 P and V). Pair unit (5, 6) shares every
    MMA between a half that attends to block 4 (window of 5) and one that does
    not (window of 6), so the second half must be untouched.

    Bars: rows that do not attend to block 4 at the forward's bar (max 1e-2,
    mean 1e-3) and finite. Rows that do: attention is linear in V, and the
    large tile's weights are rounded once to 16 bits (bf16: relative 2^-9) and,
    with bf16 output, the output once more (2^-9 of |out| <= the same scale),
    so |err| <= 1e-2 + 2^-7 * mass4 * max|v4|, mass4 = the row's attention
    weight on block 4 (the oracle's output for V = 1 on block 4, 0 elsewhere)."""
    w = Workload("bigv", 1, 2, 16 * 64, pad=("fixed", [1000]), seed=19)
    j = 4
    inp = make_inputs(w)
    ra_c, ra_o = _rand_attn_pair(w)
    for h in range(w.H):  # keep block 4 out of query block 6's random blocks
        row = list(ra_o[h, 5])
        if j in row:
            row[row.index(j)] = [x for x in range(1, w.nb - 1) if x not in (5, 6, 7, j) and x not in row][0]
            ra_o[h, 5] = row
    assert bb.rand_attn_validate(ra_o, w.H, w.L, w.block, w.r) == bb.BB_OK
    ra_c = ra_o.copy()
    v = inp["v"].clone()
    big = torch.randn(w.B, w.H, 64, 64, generator=torch.Generator().manual_seed(5))
    v[:, :, j * 64:(j + 1) * 64] = (big / big.abs().max() * vmax).to(torch.bfloat16)
    inp = dict(inp, v=v)
    got = _cuda_fwd(inp, w, ra_c, out_dtype)
    assert np.isfinite(got).all()
    want = oracle.attention(inp["q"], inp["k"], v, ra_o, inp["seq_mask"], w.block, w.r)
    ind = np.zeros(v.shape, np.float64)
    ind[:, :, j * 64:(j + 1) * 64] = 1.0
    mass = oracle.attention(inp["q"], inp["k"], ind, ra_o, inp["seq_mask"], w.block, w.r)[..., :1]
    vmax4 = float(v[:, :, j * 64:(j + 1) * 64].float().abs().max())
    err = np.abs(got.astype(np.float64) - want)
    for h in range(w.H):
        bm = oracle.block_mask(w.nb, w.r, ra_o[h], True)
        attends = np.repeat(bm[:, j], 64)          # per query row
        assert not attends[6 * 64] and attends[5 * 64], "pair (5, 6) must split on block 4"
        e_off = err[0, h, ~attends]
        assert e_off.max() <= MAX_ABS and e_off.mean() <= MEAN_ABS, (h, float(e_off.max()))
        bar = 1e-2 + 2.0 ** -7 * mass[0, h, attends] * vmax4
        assert (err[0, h, attends] <= bar).all(), (h, float((err[0, h, attends] / bar).max()))


def test_v_beyond_fp16_range_many_ranges():
    """The recompute path at L = 4096 with more work units than CTAs: eight key
    ranges per global row, each redone by the bf16 instance, which waits until
    every range is written and then merges them. Key block 0 (a global block,
    attended by every row) holds V at 1e5, so every row carries that path's
    error bar: |err| <= 1e-2 + 2^-7 * mass0 * max|v0| (mass0 = the row's weight
    on block 0). Two calls give the same bits: the merge of a row does not
    depend on which CTA does it. Heads (b 0, h 0) and (b 1, h 7) are checked
    against the oracle, every head for finiteness."""
    w = Workload("bigv_l4096", 2, 8, 4096, pad=("fixed", [4096, 3001]), seed=23)
    inp = make_inputs(w)
    ra_c, ra_o = _rand_attn_pair(w)
    v = inp["v"].clone()
    big = torch.randn(w.B, w.H, 64, 64, generator=torch.Generator().manual_seed(7))
    v[:, :, :64] = (big / big.abs().max() * 1.0e5).to(torch.bfloat16)
    inp = dict(inp, v=v)
    got = _cuda_fwd(inp, w, ra_c, torch.float32)
    again = _cuda_fwd(inp, w, ra_c, torch.float32)
    assert np.isfinite(got).all()
    assert np.array_equal(got, again)
    vmax0 = float(v[:, :, :64].float().abs().max())
    for b, h in [(0, 0), (1, 7)]:
        sl = {x: inp[x][b:b + 1, h:h + 1] for x in "qk"}
        vb = v[b:b + 1, h:h + 1]
        sm = inp["seq_mask"][b:b + 1]
        ra_h = ra_o[h:h + 1]
        want = oracle.attention(sl["q"], sl["k"], vb, ra_h, sm, w.block, w.r)
        ind = np.zeros(vb.shape, np.float64)
        ind[:, :, :64] = 1.0
        mass = oracle.attention(sl["q"], sl["k"], ind, ra_h, sm, w.block, w.r)[..., :1]
        err = np.abs(got[b:b + 1, h:h + 1].astype(np.float64) - want)
        assert (err <= 1e-2 + 2.0 ** -7 * mass * vmax0).all(), (b, h, float((err / (1e-2 + 2.0 ** -7 * mass * vmax0)).max()))


def test_out_of_range_rand_attn_is_flagged():
    w = Workload("oor", 1, 1, 16 * 64, seed=18)
    inp = make_inputs(w)
    ra = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=1)
    ra[0, 3, 1] = w.nb + 5
    q, k, v = (inp[x].cuda() for x in "qkv")
    bb.fwd(q, k, v, torch.from_numpy(ra).cuda(), None)
    assert bb.device_status() & 1
    with pytest.raises(bb.BigBirdError) as e:
        bb.fwd(q, k, v, torch.from_numpy(ra).cuda(), None, debug_checks=True)
    assert e.value.status == bb.BB_ERR_BAD_RAND_ATTN
    assert bb.device_status() == 0


def test_bounded_wait_runs_out_and_is_reported():
    """Failure detection without a fault: a wait on an mbarrier that nothing
    arrives on gives up after its limit, the host reads the timeout bit, and
    the context stays usable (a forward afterwards is correct and clean)."""
    import ctypes
    lib = bb.lib()
    assert lib.bigbird_wait_probe(0, None) == bb.BB_ERR_INVALID_ARG
    st = lib.bigbird_wait_probe(20000, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bb.BB_OK
    assert bb.device_status() == 2
    assert bb.device_status() == 0  # read-and-clear
    w = WORKLOADS["tiny_l1024"]
    inp = make_inputs(w)
    ra, ra_o = _rand_attn_pair(w)
    got = _cuda_fwd(inp, w, ra, torch.float32)
    want = oracle.attention(inp["q"], inp["k"], inp["v"], ra_o, inp["seq_mask"], w.block, w.r)
    _check(got, want, "after probe")
