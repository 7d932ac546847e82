"""Host-side library checks that need no GPU: the C ABI loads and exports every
declared symbol, the host preparation routines match the oracle bit for bit,
and argument errors come back as status codes."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import block_sparse_long_attention_b200 as bb
from block_sparse_long_attention_b200.workloads import mask_from_lengths

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_lib():
    from block_sparse_long_attention_b200 import build
    build.build()
    return bb.lib()


def _declared_functions():
    txt = open(os.path.join(ROOT, "include", "bigbird_attn.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(bigbird_\w+)\s*\(", txt)))


def test_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(bb.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


@pytest.mark.parametrize("H,L,r,seed,last_idx", [
    (2, 1024, 3, 1001, 0), (12, 4096, 3, 1002, 0), (3, 640, 1, 7, 0), (2, 2048, 5, 2**63 + 5, 0),
    (4, 4096, 3, 99, 1024), (1, 32768, 3, 1005, 0), (16, 4096, 3, 0, 0)])
def test_generator_bit_exact(H, L, r, seed, last_idx):
    got = bb.rand_attn_generate(H, L, 64, r, seed=seed, last_idx=last_idx)
    want = oracle.rand_attn_generate(H, L, 64, r, seed=seed, last_idx=last_idx)
    assert got.dtype == np.int32 and np.array_equal(got, want)
    assert bb.rand_attn_validate(got, H, L, 64, r, last_idx) == bb.BB_OK


def test_generator_errors():
    with pytest.raises(bb.BigBirdError) as e:
        bb.rand_attn_generate(1, 7 * 64, 64, 3, seed=1)
    assert e.value.status == bb.BB_ERR_INVALID_ARG
    with pytest.raises(bb.BigBirdError):
        bb.rand_attn_generate(1, 4096, 64, 3, seed=1, last_idx=256)
    with pytest.raises(bb.BigBirdError):
        bb.rand_attn_generate(1, 1000, 64, 3, seed=1)
    with pytest.raises(bb.BigBirdError):
        bb.rand_attn_generate(1, 1024, 64, 0, seed=1)


def test_validator_matches_oracle():
    H, L, r = 2, 1024, 3
    ra = oracle.rand_attn_generate(H, L, 64, r, seed=3)
    rng = np.random.default_rng(0)
    for trial in range(200):
        bad = ra.copy()
        h, row, t = rng.integers(0, H), rng.integers(0, L // 64 - 2), rng.integers(0, r)
        bad[h, row, t] = rng.integers(-1, L // 64 + 1)
        try:
            oracle.rand_attn_validate(bad, H, L, 64, r)
            want = bb.BB_OK
        except ValueError:
            want = bb.BB_ERR_BAD_RAND_ATTN
        assert bb.rand_attn_validate(bad, H, L, 64, r) == want


@pytest.mark.parametrize("vl", [[1024, 700, 130], [0, 64, 1023], [1024, 1024, 1024]])
def test_mask_prep_bit_exact(vl):
    sm = mask_from_lengths(3, 1024, vl).numpy()
    got = bb.mask_prep(sm, 64)
    want = oracle.mask_prep(sm, 64)
    for g, w in zip(got, want):
        assert g.shape == w.shape and np.array_equal(g, w)


def test_mask_prep_nonbinary_input():
    sm = np.random.default_rng(1).integers(0, 4, size=(2, 512)).astype(np.uint8)
    for g, w in zip(bb.mask_prep(sm, 64), oracle.mask_prep(sm, 64)):
        assert np.array_equal(g, w)


def test_pattern_table_bit_exact():
    H, L, r = 3, 2048, 3
    ra = oracle.rand_attn_generate(H, L, 64, r, seed=11)
    assert np.array_equal(bb.pattern_table(ra, H, L, 64, r), oracle.pattern_table(ra, H, L, 64, r))
    dup = ra.copy(); dup[0, 3, :] = 0; dup[1, 7, 1] = dup[1, 7, 0]
    assert np.array_equal(bb.pattern_table(dup, H, L, 64, r), oracle.pattern_table(dup, H, L, 64, r))
    bad = ra.copy(); bad[2, 0, 0] = L // 64
    with pytest.raises(bb.BigBirdError) as e:
        bb.pattern_table(bad, H, L, 64, r)
    assert e.value.status == bb.BB_ERR_BAD_RAND_ATTN


def test_fallback_rule_matches_oracle():
    for L in range(64, 64 * 40, 64):
        for r in (1, 2, 3, 5):
            assert bb.is_fallback(L, 64, r) == oracle.is_fallback(L, 64, r)
    with pytest.raises(bb.BigBirdError):
        bb.is_fallback(1000, 64, 3)


def test_workspace_size():
    head = 256  # unit-ticket, finished-CTA and bf16-recompute counters
    assert bb.workspace_size(1, 2, 704) == head  # fallback: no split rows
    nb = 4096 // 64
    nsplit = (nb + 7) // 8  # global rows split into ranges of 8 key blocks
    assert bb.workspace_size(4, 12, 4096) == head + 4 * 12 * nsplit * 128 * 66 * 4
    nb = 125  # a ragged last range
    assert bb.workspace_size(1, 3, nb * 64) == head + 3 * ((nb + 7) // 8) * 128 * 66 * 4
    assert bb.workspace_size(1, 1, 1000) == 0  # invalid sizes


def test_fwd_argument_errors_before_any_launch():
    lib = bb.lib()
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: every case fails argument checks first
    cases = [
        (dict(L=1000), bb.BB_ERR_INVALID_ARG),   # not a multiple of the block
        (dict(r=0), bb.BB_ERR_INVALID_ARG),      # r = 0 unsupported
        (dict(d=96), bb.BB_ERR_UNSUPPORTED),
        (dict(block=48, L=3072), bb.BB_ERR_UNSUPPORTED),
        (dict(d=128, L=1000), bb.BB_ERR_INVALID_ARG),       # the CUDA-core sizes check their arguments too
        (dict(block=32, r=0), bb.BB_ERR_INVALID_ARG),
        (dict(B=0), bb.BB_ERR_INVALID_ARG),
        (dict(r=17), bb.BB_ERR_UNSUPPORTED),
    ]
    for kw, want in cases:
        a = dict(B=1, H=2, L=4096, d=64, block=64, r=3)
        a.update(kw)
        st = lib.bigbird_attn_fwd(fake, fake, fake, fake, None, fake, a["B"], a["H"], a["L"], a["d"], a["block"],
                                  a["r"], None)
        assert st == want, (kw, st)
    # NULL q and a misaligned out pointer
    assert lib.bigbird_attn_fwd(None, fake, fake, fake, None, fake, 1, 2, 4096, 64, 64, 3, None) == bb.BB_ERR_INVALID_ARG
    assert lib.bigbird_attn_fwd(fake, fake, fake, fake, None, P(0x10008), 1, 2, 4096, 64, 64, 3, None) == bb.BB_ERR_UNSUPPORTED
    # sparse mode needs rand_attn
    assert lib.bigbird_attn_fwd(fake, fake, fake, None, None, fake, 1, 2, 4096, 64, 64, 3, None) == bb.BB_ERR_INVALID_ARG
    # forced sparse needs nb >= 5 + r
    assert lib.bigbird_attn_fwd_ex(fake, fake, fake, fake, None, fake, 1, 2, 7 * 64, 64, 64, 3, 0,
                                   bb.BB_FLAG_FORCE_SPARSE, None, 0, None) == bb.BB_ERR_INVALID_ARG
    # the other sizes (block 128 and d 128 on tensor cores, block 32 on CUDA
    # cores) check the same before any device call
    for d, block in ((64, 32), (64, 128), (128, 32), (128, 64), (128, 128)):
        L = 16 * block
        assert lib.bigbird_attn_fwd(None, fake, fake, fake, None, fake, 1, 2, L, d, block, 3, None) == \
            bb.BB_ERR_INVALID_ARG
        assert lib.bigbird_attn_fwd(fake, fake, fake, fake, None, P(0x10008), 1, 2, L, d, block, 3, None) == \
            bb.BB_ERR_UNSUPPORTED
        assert lib.bigbird_attn_fwd(fake, fake, fake, None, None, fake, 1, 2, L, d, block, 3, None) == \
            bb.BB_ERR_INVALID_ARG
        assert lib.bigbird_attn_fwd_ex(fake, fake, fake, fake, None, fake, 1, 2, 7 * block, d, block, 3, 0,
                                       bb.BB_FLAG_FORCE_SPARSE, None, 0, None) == bb.BB_ERR_INVALID_ARG
        if block == 32:
            assert bb.workspace_size(1, 2, L, d, block) == 0   # CUDA cores: no workspace
    # block 128 at d 64: 64-token tiles, nt = L / 64, the global rows split
    # into ranges of 8 tiles, one partial-result set per global block
    nt = 2048 // 64
    assert bb.workspace_size(1, 2, 2048, 64, 128) == 256 + 2 * 2 * ((nt + 7) // 8) * 128 * 66 * 4
    assert bb.workspace_size(1, 2, 8 * 128, 64, 128) == 256            # fallback: no split rows
    assert bb.workspace_size(1, 2, 22 * 128, 64, 128, r=9) == 0        # fallback wider than a unit: CUDA cores
    # d 128: partial outputs of 128 columns (plus max and sum)
    assert bb.workspace_size(1, 2, 4096, 128, 64) == 256 + 2 * 8 * 128 * 130 * 4
    assert bb.workspace_size(1, 2, 4096, 128, 128) == 256 + 2 * 2 * 8 * 128 * 130 * 4
    # the backward and the probability export take d = block = 64 only
    assert lib.bigbird_attn_probs(fake, fake, fake, fake, None, fake, fake, 1, 2, 4096, 128, 64, 3, 1, 0, None) == \
        bb.BB_ERR_UNSUPPORTED
    assert bb.status_string(bb.BB_ERR_UNSUPPORTED) == "unsupported configuration"


def test_probs_layout_and_argument_errors_before_any_launch():
    # packed layout: G full rows per head, then [nb-2, 5+r] band tiles whose
    # slot t is column t of the pattern table
    assert bb.probs_layout(4096) == (2, 62, 8)
    assert bb.probs_layout(2048, r=5) == (2, 30, 10)
    assert bb.probs_layout(704) == (11, 0, 0)                    # fallback: the whole matrix
    assert bb.probs_layout(8 * 64, force_sparse=True) == (2, 6, 8)
    ra = oracle.rand_attn_generate(2, 4096, 64, 3, seed=1)
    assert oracle.pattern_table(ra, 2, 4096, 64, 3).shape == (2, 62, 8)
    with pytest.raises(bb.BigBirdError):
        bb.probs_layout(1000)
    lib = bb.lib()
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: every case fails argument checks first
    base = dict(q=fake, k=fake, lse=fake, ra=fake, sm=None, pg=fake, pb=fake, B=1, H=2, L=4096, d=64, block=64, r=3,
                dt=bb.BB_OUT_F32, fl=0)
    cases = [
        (dict(L=1000), bb.BB_ERR_INVALID_ARG),
        (dict(r=0), bb.BB_ERR_INVALID_ARG),
        (dict(d=128), bb.BB_ERR_UNSUPPORTED),
        (dict(B=0), bb.BB_ERR_INVALID_ARG),
        (dict(lse=None), bb.BB_ERR_INVALID_ARG),
        (dict(pb=None), bb.BB_ERR_INVALID_ARG),       # the sparse mode needs the band output
        (dict(ra=None), bb.BB_ERR_INVALID_ARG),       # and rand_attn
        (dict(pg=P(0x10004)), bb.BB_ERR_UNSUPPORTED),  # misaligned output
        (dict(dt=7), bb.BB_ERR_INVALID_ARG),
        (dict(L=7 * 64, fl=bb.BB_FLAG_FORCE_SPARSE), bb.BB_ERR_INVALID_ARG),
    ]
    for kw, want in cases:
        a = dict(base)
        a.update(kw)
        st = lib.bigbird_attn_probs(a["q"], a["k"], a["lse"], a["ra"], a["sm"], a["pg"], a["pb"], a["B"], a["H"],
                                    a["L"], a["d"], a["block"], a["r"], a["dt"], a["fl"], None)
        assert st == want, (kw, st)
    assert lib.bigbird_attn_probs_dense(fake, fake, None, fake, None, fake, 1, 2, 4096, 64, 64, 3, bb.BB_OUT_F32, 0,
                                        None) == bb.BB_ERR_INVALID_ARG
    assert lib.bigbird_attn_probs_dense(fake, fake, fake, fake, None, P(0x10002), 1, 2, 4096, 64, 64, 3,
                                        bb.BB_OUT_BF16, 0, None) == bb.BB_ERR_UNSUPPORTED


@pytest.mark.parametrize("block", [32, 128])
def test_host_prep_other_block_sizes(block):
    """The pages' only knob is block_size: the host routines (generator,
    validator, masks, pattern table, fallback rule) follow the oracle bit for
    bit at other block sizes too. (The GPU kernels take block 64 only.)"""
    H, L, r = 3, 64 * block, 3
    for seed, last_idx in ((5, 0), (2**63 + 1, 0), (9, 40 * block)):
        got = bb.rand_attn_generate(H, L, block, r, seed=seed, last_idx=last_idx)
        want = oracle.rand_attn_generate(H, L, block, r, seed=seed, last_idx=last_idx)
        assert np.array_equal(got, want)
        assert bb.rand_attn_validate(got, H, L, block, r, last_idx) == bb.BB_OK
    ra = oracle.rand_attn_generate(H, L, block, r, seed=7)
    assert np.array_equal(bb.pattern_table(ra, H, L, block, r), oracle.pattern_table(ra, H, L, block, r))
    sm = mask_from_lengths(2, L, [L - 3 * block - 5, block]).numpy()
    for g, w in zip(bb.mask_prep(sm, block), oracle.mask_prep(sm, block)):
        assert g.shape == w.shape and np.array_equal(g, w)
    for LL in range(block, block * 30, block):
        assert bb.is_fallback(LL, block, r) == oracle.is_fallback(LL, block, r)
    assert bb.is_fallback((5 + 2 * r) * block, block, r) and not bb.is_fallback((6 + 2 * r) * block, block, r)
