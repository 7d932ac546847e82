"""Attention probabilities (bigbird_attn_probs and bigbird_attn_probs_dense
through the C ABI) against the oracle's fp64 weight matrix.

The GPU forms p = exp2(x), x = (s + bias) log2(e) / sqrt(d) - lse log2(e), in
fp32: s is the tensor cores' fp32 sum of exact bf16 products and lse the GPU
forward's own log-sum-exp (fp32 sums of unrounded exponentials, ~1e-6
absolute). For |x| up to ~60 the fp32 roundings of x stay below ~5e-6 (log2
units) and ex2.approx adds ~2 ulp, so |dp| <~ 5e-6 p. Bars per element:
|err| <= 2e-5 p + 1e-12 with fp32 output, 4e-3 p + 1e-12 with bf16 output
(8 significant bits: rounding to nearest moves a value by up to 2^-8 of
itself). Rows whose keys are all padded have lse near
-10000, where fp32 resolves ~1e-3: 4e-3 p there. Zeros (outside the pattern,
padded keys of rows with a valid key, band slots past the end of a row's
list) therefore have to be exact.
"""

import numpy as np
import pytest
import torch

import oracle
import block_sparse_long_attention_b200 as bb
from block_sparse_long_attention_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

REL_F32, REL_BF16, REL_ALL_PADDED, ABS_FLOOR = 2e-5, 4e-3, 4e-3, 1e-12


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_attention_b200 import build
    build.build()
    bb.device_status()
    yield


def _sparse(w, force=False):
    return force or not oracle.is_fallback(w.L, w.block, w.r)


def _gpu_lse(inp, w, ra, force=False):
    q, k, v = (inp[x].cuda() for x in "qkv")
    sm = None if inp["seq_mask"] is None else inp["seq_mask"].cuda()
    ra_d = None if ra is None else torch.from_numpy(np.ascontiguousarray(ra)).cuda()
    _, lse = bb.fwd_train(q, k, v, ra_d, sm, block=w.block, r=w.r, out_dtype=torch.float32, force_sparse=force)
    return q, k, lse, ra_d, sm


def _pack(P, ra, w, force=False):
    """The oracle's [B, H, L, L] matrix in the packed layout (global rows, band tiles)."""
    B, H, L = w.B, w.H, w.L
    nb = L // 64
    if not _sparse(w, force):
        return P.reshape(B, H, nb, 64, L), None
    glob = np.stack([P[:, :, :64, :], P[:, :, L - 64:, :]], axis=2)
    pt = oracle.pattern_table(ra, H, L, 64, w.r)
    band = np.zeros((B, H, nb - 2, 5 + w.r, 64, 64))
    for h in range(H):
        for i in range(1, nb - 1):
            for t, kb in enumerate(pt[h, i - 1]):
                if kb >= 0:
                    band[:, h, i - 1, t] = P[:, h, i * 64:(i + 1) * 64, kb * 64:(kb + 1) * 64]
    return glob, band


def _close(got, want, rel, what, rows_rel=None):
    got = got.astype(np.float64)
    bar = rel * np.abs(want) + ABS_FLOOR
    if rows_rel is not None:
        bar = np.maximum(bar, rows_rel * np.abs(want) + ABS_FLOOR)
    bad = np.abs(got - want) > bar
    assert np.isfinite(got).all(), what
    assert not bad.any(), (what, int(bad.sum()), float(np.abs(got - want).max()))
    nz = want != 0
    return float((np.abs(got - want)[nz] / want[nz]).max()) if nz.any() else 0.0


SMALL = [
    WORKLOADS["tiny_l1024"],
    Workload("pairs_odd_tail", 1, 2, 13 * 64, pad=("fixed", [800]), seed=7),
    Workload("split3_padded", 2, 3, 24 * 64, pad=("fixed", [1000, 1536]), seed=8),
    Workload("ragged_split", 1, 2, 21 * 64, pad=("fixed", [1300]), seed=10),
    Workload("fallback_704", 2, 2, 704, pad=("fixed", [700, 100]), seed=11),
    Workload("fallback_one_block", 1, 2, 64, seed=12),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_probs_all_elements(w, dtype):
    inp = make_inputs(w)
    ra = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed) if _sparse(w) else None
    q, k, lse, ra_d, sm = _gpu_lse(inp, w, ra)
    pg, pb = bb.probs(q, k, lse, ra_d, sm, block=w.block, r=w.r, out_dtype=dtype)
    pd = bb.probs_dense(q, k, lse, ra_d, sm, block=w.block, r=w.r, out_dtype=dtype)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    P = oracle.attention_probs(inp["q"], inp["k"], ra, inp["seq_mask"], w.block, w.r)
    glob, band = _pack(P, ra, w)
    rel = REL_F32 if dtype == torch.float32 else REL_BF16
    _close(pg.float().cpu().numpy(), glob, rel, "global rows")
    if band is None:
        assert pb is None
    else:
        _close(pb.float().cpu().numpy(), band, rel, "band tiles")
    _close(pd.float().cpu().numpy(), P, rel, "dense")


def test_probs_forced_sparse_and_set_semantics():
    """BB_FLAG_FORCE_SPARSE at nb = 5 + r; duplicate and window-overlapping
    random entries (their list is shorter: the band slots past its end are
    zero); a sequence with every key padded."""
    w = Workload("forced", 1, 2, 8 * 64, seed=14)
    inp = make_inputs(w)
    nb = w.L // 64
    ra = np.zeros((w.H, nb - 2, w.r), dtype=np.int32)
    for h in range(w.H):
        for i in range(1, nb - 1):
            rest = [j for j in range(1, nb - 1) if abs(j - i) > 1]
            ra[h, i - 1] = (rest + [rest[0]] * w.r)[:w.r]
    q, k, lse, ra_d, sm = _gpu_lse(inp, w, ra, force=True)
    pg, pb = bb.probs(q, k, lse, ra_d, sm, block=64, r=w.r, force_sparse=True)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    glob, band = _pack(oracle.attention_probs(inp["q"], inp["k"], ra, None, 64, w.r, force_sparse=True), ra, w, True)
    _close(pg.cpu().numpy(), glob, REL_F32, "forced global")
    _close(pb.cpu().numpy(), band, REL_F32, "forced band")

    w = Workload("edge", 2, 2, 20 * 64, pad=("fixed", [1280, 0]), seed=17)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=4)
    ra[0] = 0                         # eval-mode all-zero adjacency: duplicates of the global block
    ra[1, 5, :] = ra[1, 5, 0]         # a repeated entry
    ra[1, 9, 0] = 10                  # inside the window of row 10
    q, k, lse, ra_d, sm = _gpu_lse(inp, w, ra)
    pg, pb = bb.probs(q, k, lse, ra_d, sm, block=64, r=w.r)
    pd = bb.probs_dense(q, k, lse, ra_d, sm, block=64, r=w.r)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    P = oracle.attention_probs(inp["q"], inp["k"], ra, inp["seq_mask"], 64, w.r)
    glob, band = _pack(P, ra, w)
    # sequence 1 has every key padded: its rows get the looser bar
    rows_rel = np.zeros((w.B, 1, 1, 1))
    rows_rel[1] = REL_ALL_PADDED
    _close(pd.cpu().numpy(), P, REL_F32, "edge dense", rows_rel=rows_rel)
    _close(pg.cpu().numpy(), glob, REL_F32, "edge global", rows_rel=rows_rel[..., None])
    _close(pb.cpu().numpy(), band, REL_F32, "edge band", rows_rel=rows_rel[..., None, None])
    assert np.all(pb[0, 0].cpu().numpy()[:, 5:] == 0.0)   # row lists of head 0 hold 5 blocks: slots 5.. are zero


@pytest.mark.parametrize("name", ["bigbird_base_l4096", "extreme_l32768"])
def test_probs_full_size_sampled(name):
    """The packed export at full size: sampled rows of every (b, h) against
    the oracle, and every row's weights sum to one."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    ra = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
    q, k, lse, ra_d, sm = _gpu_lse(inp, w, ra)
    pg, pb = bb.probs(q, k, lse, ra_d, sm, block=64, r=w.r)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    L, nb = w.L, w.L // 64
    # row sums over the packed tiles (every row has a valid key here)
    sums = torch.cat([pg.sum(dim=-1).reshape(w.B, w.H, 2, 64), pb.sum(dim=(3, 5)).reshape(w.B, w.H, nb - 2, 64)], 2)
    assert float((sums.double() - 1.0).abs().max()) < 1e-4
    pt = oracle.pattern_table(ra, w.H, L, 64, w.r)
    rng = np.random.default_rng(5)
    worst = 0.0
    for b in range(w.B):
        for h in range(w.H):
            blocks = [0, nb - 1] + [int(x) for x in rng.integers(1, nb - 1, size=3)]
            rows = [blk * 64 + int(rng.integers(64)) for blk in blocks]
            want = oracle.attention_probs_rows(inp["q"], inp["k"], ra, inp["seq_mask"], 64, w.r, b, h, rows)
            for n, t in enumerate(rows):
                i, qq = divmod(t, 64)
                if i in (0, nb - 1):
                    got = pg[b, h, 0 if i == 0 else 1, qq].cpu().numpy()
                    worst = max(worst, _close(got, want[n], REL_F32, (name, b, h, t)))
                else:
                    tiles = pb[b, h, i - 1, :, qq].cpu().numpy()   # [5+r, 64]
                    for s, kb in enumerate(pt[h, i - 1]):
                        seg = want[n, kb * 64:(kb + 1) * 64] if kb >= 0 else np.zeros(64)
                        worst = max(worst, _close(tiles[s], seg, REL_F32, (name, b, h, t, s)))
                    listed = [kb for kb in pt[h, i - 1] if kb >= 0]
                    rest = np.delete(want[n].reshape(nb, 64), listed, axis=0)
                    assert np.all(rest == 0.0)
    print(f"{name}: worst relative error {worst:.3g}")


def test_probs_dense_matches_packed_at_full_size():
    """At the BigBird-base size the dense matrix holds exactly the packed
    tiles (bit for bit: the same arithmetic) and zeros elsewhere."""
    w = WORKLOADS["bigbird_base_l4096"]
    inp = make_inputs(w)
    ra = bb.rand_attn_generate(w.H, w.L, w.block, w.r, seed=w.seed)
    q, k, lse, ra_d, sm = _gpu_lse(inp, w, ra)
    pg, pb = bb.probs(q, k, lse, ra_d, sm, block=64, r=w.r, out_dtype=torch.bfloat16)
    pd = bb.probs_dense(q, k, lse, ra_d, sm, block=64, r=w.r, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    L, nb = w.L, w.L // 64
    assert torch.equal(pd[:, :, :64], pg[:, :, 0]) and torch.equal(pd[:, :, L - 64:], pg[:, :, 1])
    pt_np = oracle.pattern_table(ra, w.H, L, 64, w.r)
    pt = torch.from_numpy(pt_np).long().cuda()   # [H, nb-2, 5+r]
    blocks = pd[:, :, 64:L - 64].reshape(w.B, w.H, nb - 2, 64, nb, 64)
    listed_np = np.zeros((w.H, nb - 2, nb), dtype=bool)
    for h in range(w.H):
        for i in range(nb - 2):
            listed_np[h, i, pt_np[h, i][pt_np[h, i] >= 0]] = True
    listed = torch.from_numpy(listed_np).cuda()
    for s in range(5 + w.r):
        kb = pt[:, :, s].clamp(min=0)                     # [H, nb-2]
        idx = kb[None, :, :, None, None, None].expand(w.B, w.H, nb - 2, 64, 1, 64)
        tile = torch.gather(blocks, 4, idx).squeeze(4)     # [B, H, nb-2, 64, 64]
        valid = (pt[:, :, s] >= 0)[None, :, :, None, None]
        assert torch.equal(torch.where(valid, tile, 0), torch.where(valid, pb[:, :, :, s], 0))
    off = (~listed)[None, :, :, None, :, None].expand_as(blocks)
    assert float(blocks.float().abs()[off].max()) == 0.0


def test_probs_out_of_range_rand_attn_is_flagged():
    w = Workload("oor", 1, 1, 16 * 64, seed=18)
    inp = make_inputs(w)
    ra = oracle.rand_attn_generate(w.H, w.L, w.block, w.r, seed=2)
    q, k, lse, ra_d, sm = _gpu_lse(inp, w, ra)
    bb.device_status()
    ra_d[0, 3, 1] = 999
    bb.probs(q, k, lse, ra_d, sm, block=64, r=w.r)
    assert bb.device_status() & 1


def test_probs_max_r_with_duplicates():
    """r = 16, the largest supported (21 candidate key blocks per query
    block), with entries 10..15 of every row repeating blocks listed before
    them (the row's first entry, a global block, its window block, the
    previous row's entry): every element of the packed and dense layouts
    against the oracle's weights (set semantics: a repeated block is listed
    once) [TFG-BigBird, section "随机块掩码是如何生成的"]."""
    nb = 40
    w = Workload("probs_max_r", 1, 2, nb * 64, r=16, pad=("fixed", [nb * 64 - 150]), seed=23)
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
    q, k, lse, ra_d, sm = _gpu_lse(inp, w, ra)
    pg, pb = bb.probs(q, k, lse, ra_d, sm, block=64, r=w.r)
    pd = bb.probs_dense(q, k, lse, ra_d, sm, block=64, r=w.r)
    torch.cuda.synchronize()
    assert bb.device_status() == 0
    P = oracle.attention_probs(inp["q"], inp["k"], ra, inp["seq_mask"], w.block, w.r)
    glob, band = _pack(P, ra, w)
    _close(pg.cpu().numpy(), glob, REL_F32, "global rows")
    _close(pb.cpu().numpy(), band, REL_F32, "band tiles")
    _close(pd.cpu().numpy(), P, REL_F32, "dense")
