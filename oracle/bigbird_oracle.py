"""Plain fp64 CPU oracle of BigBird ITC block-sparse attention (forward, its
attention probabilities, and the backward).

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module. Every function below is a direct, unoptimised statement of
what the pages define; there is no blocking, fusion or reordering beyond the
row chunking needed to keep an [L, L] score matrix in memory.

What the method computes (the plain definition this oracle writes out)
---------------------------------------------------------------------
Q, K, V of shape [B, H, L, d] are cut into nb = L / block query and key blocks
[TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力"]. Query block i
attends to the key blocks of a boolean block mask BM[i, :]:

* the first and last query blocks (0 and nb-1) attend to every key block
  (global rows) [TFG-BigBird, same section; HF-Pegasus, section "三类注意力组合"];
* every other query block i attends to the two global key blocks 0 and nb-1,
  the 3-block sliding window {i-1, i, i+1}, and the r random key blocks
  rand_attn[h][i-1][0..r) [TFG-BigBird, same section and section
  "随机块掩码是如何生成的"; HF-Pegasus, section "三类注意力组合"].

The block mask is expanded to a token mask M[q, k] = BM[q // block, k // block].
Scores are s[q, k] = (q . k) / sqrt(d) + bias[k], with bias[k] = -10000 for a
padded key and 0 otherwise, wherever M is true, and -inf (absent) elsewhere
[TFG-BigBird, section "BigBird：从二次方注意力到线性稀疏注意力": masked positions
get -10000 before the softmax]. Then p = softmax over k, out[q] = sum_k p v_k.

When nb <= 5 + 2r the method falls back to full attention
[HF-Pegasus, section "序列过短时的自动回退": (5 + 2*3) * 64 = 704 tokens at the
defaults]. A length that is not a multiple of block is an error
[HF-Pegasus, section "序列长度的块对齐要求"]; r = 0 is unsupported
[HF-Pegasus, section "使用限制与注意事项"].

Readings where the pages leave a step open:
the random blocks of a row are a *set* (a duplicated or window-overlapping
entry adds nothing); the second rows (1 and nb-2) follow the same three rules;
the -10000 bias applies to padded keys only and is added after the 1/sqrt(d)
scaling; the random-block generator is a seeded SplitMix64 stream driving a
partial Fisher-Yates shuffle of the candidate pool.
"""

from __future__ import annotations

import math

import numpy as np

BIAS_MASKED = -10000.0
"""Additive bias of a masked key [TFG-BigBird, "BigBird：从二次方注意力到线性稀疏注意力"]."""

_MASK64 = (1 << 64) - 1
_SM64_GAMMA = 0x9E3779B97F4A7C15
_ROW_COUNTER_SHIFT = 20  # draws of one (head, row) use counters base+1 .. base+2^20


# --------------------------------------------------------------------------
# Argument rules
# --------------------------------------------------------------------------

def check_shape(L: int, block: int, r: int) -> int:
    """Return nb = L // block after the pages' argument rules.

    L must be a positive multiple of block [HF-Pegasus, "序列长度的块对齐要求"];
    r must be >= 1 [HF-Pegasus, "使用限制与注意事项": num_random_blocks = 0 is not
    supported].
    """
    if block <= 0 or L <= 0:
        raise ValueError("L and block must be positive")
    if L % block != 0:
        raise ValueError(f"sequence length {L} is not a multiple of block size {block}")
    if r < 1:
        raise ValueError("num_random_blocks must be >= 1")
    return L // block


def is_fallback(L: int, block: int, r: int) -> bool:
    """True when the method runs full attention instead of the sparse pattern.

    [HF-Pegasus, "序列过短时的自动回退"]: a sequence no longer than
    (5 + 2 r) * block tokens switches to full attention.
    """
    nb = check_shape(L, block, r)
    return nb <= 5 + 2 * r


# --------------------------------------------------------------------------
# The random-block generator (one counter-based generator, defined here from
# its published definition; the product implements the same definition on its
# own side).
# --------------------------------------------------------------------------

def splitmix64_mix(z: int) -> int:
    """SplitMix64 output function (Steele, Lea & Flood, OOPSLA 2014; the
    constants are those of Vigna's public-domain splitmix64.c)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def splitmix64_output(seed: int, n: int) -> int:
    """n-th output (n >= 1) of a SplitMix64 stream whose state starts at seed.

    The state after n steps is seed + n * gamma (mod 2^64), so the generator is
    counter based: any draw can be computed on its own.
    """
    return splitmix64_mix((seed + n * _SM64_GAMMA) & _MASK64)


def _candidate_pool(i: int, nb: int, block: int, last_idx: int) -> list[int]:
    """Random-block candidates of query-block row i (1 <= i <= nb-2).

    [TFG-BigBird, "随机块掩码是如何生成的"]: candidates are the middle blocks
    (first and last removed) minus the row's own window blocks; with a
    last_idx cap only blocks lying wholly before token last_idx qualify.
    """
    pool = []
    for j in range(1, nb - 1):
        if i - 1 <= j <= i + 1:
            continue
        if last_idx > 0 and (j + 1) * block > last_idx:
            continue
        pool.append(j)
    return pool


def rand_attn_generate(H: int, L: int, block: int, r: int, seed: int,
                       last_idx: int = 0) -> np.ndarray:
    """Per-head random adjacency rand_attn[H, nb-2, r] (int32).

    Row i-1 holds the random key blocks of query block i (1 <= i <= nb-2)
    [TFG-BigBird, "随机块掩码是如何生成的": one row per middle block, the first
    from_seq_length // block_size - 2 rows are used]. Each row is the first r
    entries of a uniformly random permutation of the row's candidate pool
    (the page permutes the pool with numpy; the permutation here is a partial
    Fisher-Yates shuffle driven by SplitMix64, bounded draws by rejection).

    Draw t of row (h, i) uses counter ((h * (nb-2) + i-1) << 20) + 1 + t'
    where t' counts draws (rejections included) within that row.
    """
    nb = check_shape(L, block, r)
    if H <= 0:
        raise ValueError("H must be positive")
    seed &= _MASK64
    out = np.zeros((H, max(nb - 2, 0), r), dtype=np.int32)
    for h in range(H):
        for i in range(1, nb - 1):
            pool = _candidate_pool(i, nb, block, last_idx)
            n = len(pool)
            if n < r:
                raise ValueError(f"row {i}: only {n} random-block candidates for r={r}")
            ctr = (h * (nb - 2) + (i - 1)) << _ROW_COUNTER_SHIFT
            for t in range(r):
                bound = n - t
                # Accept u in [thresh, 2^64): a range whose size is a multiple of bound.
                thresh = ((1 << 64) - bound) % bound
                while True:
                    ctr += 1
                    u = splitmix64_output(seed, ctr)
                    if u >= thresh:
                        break
                j = t + (u % bound)
                pool[t], pool[j] = pool[j], pool[t]
                out[h, i - 1, t] = pool[t]
    return out


def rand_attn_validate(rand_attn: np.ndarray, H: int, L: int, block: int, r: int,
                       last_idx: int = 0) -> None:
    """Raise ValueError unless rand_attn is what the generator rule allows:
    shape [H, nb-2, r], every entry a candidate of its row (a middle block
    outside the row's window, before last_idx if capped), entries distinct.
    [TFG-BigBird, "随机块掩码是如何生成的": random blocks never overlap the window.]
    """
    nb = check_shape(L, block, r)
    ra = np.asarray(rand_attn)
    if ra.shape != (H, nb - 2, r):
        raise ValueError(f"rand_attn shape {ra.shape} != {(H, nb - 2, r)}")
    for h in range(H):
        for i in range(1, nb - 1):
            row = [int(x) for x in ra[h, i - 1]]
            allowed = set(_candidate_pool(i, nb, block, last_idx))
            if len(set(row)) != r:
                raise ValueError(f"head {h} row {i}: duplicate random blocks {row}")
            for x in row:
                if x not in allowed:
                    raise ValueError(f"head {h} row {i}: block {x} is not a candidate")


# --------------------------------------------------------------------------
# The attention pattern
# --------------------------------------------------------------------------

def block_mask(nb: int, r: int, ra_h: np.ndarray | None, sparse: bool) -> np.ndarray:
    """Boolean [nb, nb] block mask BM of one head.

    Full (all true) in the fallback [HF-Pegasus, "序列过短时的自动回退"].
    Otherwise: rows 0 and nb-1 all true (global rows); column 0 and nb-1 true
    for every row (global blocks); row i in [1, nb-2] also has its window
    i-1, i, i+1 and its random blocks ra_h[i-1, :] [TFG-BigBird,
    "BigBird：从二次方注意力到线性稀疏注意力"; HF-Pegasus, "三类注意力组合"].
    """
    if not sparse:
        return np.ones((nb, nb), dtype=bool)
    bm = np.zeros((nb, nb), dtype=bool)
    bm[0, :] = True
    bm[nb - 1, :] = True
    bm[:, 0] = True
    bm[:, nb - 1] = True
    for i in range(1, nb - 1):
        bm[i, i - 1:i + 2] = True
        for j in ra_h[i - 1]:
            j = int(j)
            if not 0 <= j < nb:
                raise ValueError(f"random block {j} out of range [0, {nb})")
            bm[i, j] = True
    return bm


def _mode(L: int, block: int, r: int, force_sparse: bool) -> tuple[int, bool]:
    nb = check_shape(L, block, r)
    sparse = force_sparse or nb > 5 + 2 * r
    if sparse and nb < 5 + r:
        raise ValueError(f"sparse pattern needs nb >= 5 + r, got nb={nb}")
    return nb, sparse


def _as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor (any dtype) -> exact fp64 values
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _key_bias(seq_mask, b: int, L: int) -> np.ndarray:
    if seq_mask is None:
        return np.zeros(L, dtype=np.float64)
    m = np.asarray(seq_mask[b]).astype(bool)
    return np.where(m, 0.0, BIAS_MASKED)


def _masked_softmax_rows(qr: np.ndarray, k: np.ndarray, v: np.ndarray,
                         allowed: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(d) + bias, restricted to allowed) @ v, in fp64."""
    d = qr.shape[-1]
    s = (qr @ k.T) / math.sqrt(d) + bias[None, :]
    s = np.where(allowed, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


def attention(q, k, v, rand_attn, seq_mask, block: int, r: int,
              force_sparse: bool = False) -> np.ndarray:
    """BigBird ITC attention forward in fp64: returns out[B, H, L, d].

    q, k, v: [B, H, L, d] (numpy or torch, any float dtype; bf16 inputs are
    used at their exact values). rand_attn: [H, nb-2, r] int (ignored in the
    fallback). seq_mask: [B, L] with nonzero = valid key, or None.
    force_sparse applies the sparse pattern even when nb <= 5 + 2r.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, L, d = q.shape
    nb, sparse = _mode(L, block, r, force_sparse)
    tok_blk = np.arange(L) // block
    chunk = max(block, (1 << 22) // L // block * block)
    out = np.empty((B, H, L, d), dtype=np.float64)
    for b in range(B):
        bias = _key_bias(seq_mask, b, L)
        for h in range(H):
            bm = block_mask(nb, r, None if rand_attn is None else np.asarray(rand_attn)[h], sparse)
            for r0 in range(0, L, chunk):
                rows = np.arange(r0, min(L, r0 + chunk))
                allowed = bm[tok_blk[rows]][:, tok_blk]
                out[b, h, rows] = _masked_softmax_rows(q[b, h, rows], k[b, h], v[b, h], allowed, bias)
    return out


def attention_rows(q, k, v, rand_attn, seq_mask, block: int, r: int, b: int, h: int,
                   rows, force_sparse: bool = False) -> np.ndarray:
    """The same definition as attention(), evaluated on selected query rows
    (token indices) of one (b, h): returns [len(rows), d] in fp64."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    L = q.shape[2]
    nb, sparse = _mode(L, block, r, force_sparse)
    rows = np.asarray(rows, dtype=np.int64)
    tok_blk = np.arange(L) // block
    bm = block_mask(nb, r, None if rand_attn is None else np.asarray(rand_attn)[h], sparse)
    allowed = bm[tok_blk[rows]][:, tok_blk]
    return _masked_softmax_rows(q[b, h, rows], k[b, h], v[b, h], allowed, _key_bias(seq_mask, b, L))


def _row_key_blocks(i: int, nb: int, ra_h, sparse: bool) -> list[int]:
    """Key blocks of query block i, straight from the three rules (no BM)."""
    if not sparse or i == 0 or i == nb - 1:
        return list(range(nb))
    blocks = {0, nb - 1, i - 1, i, i + 1}
    blocks.update(int(x) for x in ra_h[i - 1])
    return sorted(blocks)


def brute_force_rows(q, k, v, rand_attn, seq_mask, block: int, r: int, b: int, h: int,
                     rows, force_sparse: bool = False) -> np.ndarray:
    """Per-query gather: for each query token, list its keys from the rules,
    then softmax over that list alone. Independent of block_mask(); used to pin
    the dense-mask oracle."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    L, d = q.shape[2], q.shape[3]
    nb, sparse = _mode(L, block, r, force_sparse)
    ra_h = None if rand_attn is None else np.asarray(rand_attn)[h]
    mask = None if seq_mask is None else np.asarray(seq_mask[b]).astype(bool)
    res = np.empty((len(rows), d), dtype=np.float64)
    for n, t in enumerate(rows):
        keys = []
        for j in _row_key_blocks(int(t) // block, nb, ra_h, sparse):
            keys.extend(range(j * block, (j + 1) * block))
        keys = np.asarray(keys)
        logits = np.array([float(np.dot(q[b, h, t], k[b, h, kk])) for kk in keys]) / math.sqrt(d)
        if mask is not None:
            logits = logits + np.where(mask[keys], 0.0, BIAS_MASKED)
        w = np.exp(logits - logits.max())
        w = w / w.sum()
        res[n] = w @ v[b, h, keys]
    return res


# --------------------------------------------------------------------------
# Host-side tables: masks and pattern
# --------------------------------------------------------------------------

def mask_prep(seq_mask: np.ndarray, block: int):
    """The four masks of the BigBirdMasks layer [TFG-BigBird, "随机块掩码是如何生成的"]:

    * blocked [B, nb, block]   : the [B, L] mask cut into blocks;
    * band    [B, nb-4, block, 3*block]: for middle query block i in [2, nb-3],
      band[b, i-2, x, w*block + y] = mask[b, i*block + x] * mask[b, (i-1+w)*block + y],
      the outer product of the query block with its 3-block window;
    * from_mask [B, L], to_mask [B, L]: the query-side and key-side masks.
    All uint8 (0/1).
    """
    m = (np.asarray(seq_mask) != 0).astype(np.uint8)
    B, L = m.shape
    if L % block:
        raise ValueError("L is not a multiple of block")
    nb = L // block
    blocked = m.reshape(B, nb, block).copy()
    nmid = max(nb - 4, 0)
    band = np.zeros((B, nmid, block, 3 * block), dtype=np.uint8)
    for w in range(3):
        frm = blocked[:, 2:2 + nmid, :, None]
        to = blocked[:, 1 + w:1 + w + nmid, None, :]
        band[:, :, :, w * block:(w + 1) * block] = frm * to
    return blocked, band, m.copy(), m.copy()


def pattern_table(rand_attn: np.ndarray, H: int, L: int, block: int, r: int) -> np.ndarray:
    """Sorted distinct key blocks of each non-global query block row of the
    sparse pattern: [H, nb-2, 5+r] int32, row i-1 for query block i, padded
    with -1. (Rows 0 and nb-1 attend to every block and are not listed.)"""
    nb = check_shape(L, block, r)
    ra = np.asarray(rand_attn)
    out = np.full((H, nb - 2, 5 + r), -1, dtype=np.int32)
    for h in range(H):
        bm = block_mask(nb, r, ra[h], True)
        for i in range(1, nb - 1):
            blocks = np.nonzero(bm[i])[0]
            out[h, i - 1, :len(blocks)] = blocks
    return out


# --------------------------------------------------------------------------
# Attention probabilities (the output_attentions path)
# --------------------------------------------------------------------------

def attention_probs(q, k, rand_attn, seq_mask, block: int, r: int, force_sparse: bool = False) -> np.ndarray:
    """The attention weights as the full matrix, probs[B, H, L, L] in fp64.

    The block-sparse model computes the weights of each row group and writes
    them back into a full (batch, heads, L, L) matrix, every position outside
    the pattern left at zero [HF-Pegasus, section "三类注意力组合": four
    scatter_ calls]; that matrix is mostly zeros and carries no gradient
    [HF-Pegasus, section "使用限制与注意事项"]. Entry [b, h, q, k] is the
    softmax weight of key k in row q (the same scores as attention()), and
    exactly 0 where k is outside the row's pattern.
    """
    q, k = _as_f64(q), _as_f64(k)
    B, H, L, d = q.shape
    nb, sparse = _mode(L, block, r, force_sparse)
    tok_blk = np.arange(L) // block
    out = np.zeros((B, H, L, L), dtype=np.float64)
    for b in range(B):
        bias = _key_bias(seq_mask, b, L)
        for h in range(H):
            bm = block_mask(nb, r, None if rand_attn is None else np.asarray(rand_attn)[h], sparse)
            out[b, h] = _probs_of_rows(q[b, h], k[b, h], bm[tok_blk][:, tok_blk], bias)
    return out


def attention_probs_rows(q, k, rand_attn, seq_mask, block: int, r: int, b: int, h: int, rows,
                         force_sparse: bool = False) -> np.ndarray:
    """Rows of attention_probs() for one (b, h): [len(rows), L] fp64."""
    q, k = _as_f64(q), _as_f64(k)
    L = q.shape[2]
    nb, sparse = _mode(L, block, r, force_sparse)
    rows = np.asarray(rows, dtype=np.int64)
    tok_blk = np.arange(L) // block
    bm = block_mask(nb, r, None if rand_attn is None else np.asarray(rand_attn)[h], sparse)
    return _probs_of_rows(q[b, h, rows], k[b, h], bm[tok_blk[rows]][:, tok_blk], _key_bias(seq_mask, b, L))


def _probs_of_rows(qr: np.ndarray, k: np.ndarray, allowed: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """Softmax weights of the rows qr over the allowed keys; 0 elsewhere."""
    s = (qr @ k.T) / math.sqrt(qr.shape[-1]) + bias[None, :]
    s = np.where(allowed, s, -np.inf)
    w = np.exp(s - s.max(axis=1, keepdims=True))   # exp(-inf) = 0 outside the pattern
    return w / w.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------
# Backward pass (gradients of the same definition)
# --------------------------------------------------------------------------

def attention_lse(q, k, rand_attn, seq_mask, block: int, r: int, force_sparse: bool = False) -> np.ndarray:
    """Natural-log log-sum-exp of each row's scores, lse[B, H, L] in fp64:
    log sum_k exp(s[q, k]) over the row's attended keys (the softmax
    normaliser the backward pass recomputes P from)."""
    q, k = _as_f64(q), _as_f64(k)
    B, H, L, d = q.shape
    nb, sparse = _mode(L, block, r, force_sparse)
    tok_blk = np.arange(L) // block
    out = np.empty((B, H, L), dtype=np.float64)
    for b in range(B):
        bias = _key_bias(seq_mask, b, L)
        for h in range(H):
            bm = block_mask(nb, r, None if rand_attn is None else np.asarray(rand_attn)[h], sparse)
            allowed = bm[tok_blk][:, tok_blk]
            s = (q[b, h] @ k[b, h].T) / math.sqrt(d) + bias[None, :]
            s = np.where(allowed, s, -np.inf)
            m = s.max(axis=1)
            out[b, h] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    return out


def attention_backward(q, k, v, rand_attn, seq_mask, block: int, r: int, dout,
                       force_sparse: bool = False):
    """Gradients (dq, dk, dv), each [B, H, L, d] fp64, of the scalar
    sum(dout * attention(q, k, v, ...)).

    Plain chain rule through the masked softmax of each row: with
    p = softmax(s), s = q k^T / sqrt(d) + bias (bias is a constant),
    dv = p^T dout, dp = dout v^T, ds = p * (dp - rowsum(dp * p)),
    dq = ds k / sqrt(d), dk = ds^T q / sqrt(d). Keys outside a row's pattern
    have p = 0 and receive nothing from it.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    B, H, L, d = q.shape
    nb, sparse = _mode(L, block, r, force_sparse)
    tok_blk = np.arange(L) // block
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    c = 1.0 / math.sqrt(d)
    for b in range(B):
        bias = _key_bias(seq_mask, b, L)
        for h in range(H):
            bm = block_mask(nb, r, None if rand_attn is None else np.asarray(rand_attn)[h], sparse)
            allowed = bm[tok_blk][:, tok_blk]
            s = (q[b, h] @ k[b, h].T) * c + bias[None, :]
            s = np.where(allowed, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            dv[b, h] = p.T @ do[b, h]
            dp = do[b, h] @ v[b, h].T
            ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
            dq[b, h] = ds @ k[b, h] * c
            dk[b, h] = ds.T @ q[b, h] * c
    return dq, dk, dv


def backward_flops(B: int, H: int, L: int, d: int, block: int, r: int) -> float:
    """Algorithmic FLOPs of one backward: 10 * B * H * L * keys_per_row * d
    (2 each for recomputing q k^T, dout v^T, p^T dout, ds k and ds^T q)."""
    return 10.0 * B * H * L * keys_per_row(L, block, r) * d


# --------------------------------------------------------------------------
# Work accounting (the metric's FLOP count)
# --------------------------------------------------------------------------

def keys_per_row(L: int, block: int, r: int, rand_attn=None, force_sparse: bool = False) -> float:
    """Average number of attended keys per query row (padded keys included).

    Without rand_attn the nominal count of a generator-valid pattern is used:
    rows 0, nb-1 see L keys, rows 1, nb-2 see (4 + r) blocks, the others 5 + r.
    """
    nb, sparse = _mode(L, block, r, force_sparse)
    if not sparse:
        return float(L)
    if rand_attn is None:
        pairs_blocks = 2 * nb + 2 * (4 + r) + (nb - 4) * (5 + r)
        return pairs_blocks * block * block / L
    ra = np.asarray(rand_attn)
    tot = 0
    for h in range(ra.shape[0]):
        tot += int(block_mask(nb, r, ra[h], True).sum())
    return tot / ra.shape[0] * block * block / L


def sparse_flops(B: int, H: int, L: int, d: int, block: int, r: int) -> float:
    """Algorithmic FLOPs of one forward: 4 * B * H * L * keys_per_row * d
    (2 for Q K^T, 2 for P V, per attended pair and head dimension)."""
    return 4.0 * B * H * L * keys_per_row(L, block, r) * d
