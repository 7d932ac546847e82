"""Seeded synthetic workloads: the inputs both the CUDA path and the oracle see.

This module draws inputs only (Q, K, V values and the padding mask). It holds
none of the attention arithmetic and none of the random-block selection: each
side derives rand_attn from the seed with its own implementation of the same
generator definition.

Workloads (the BigBird-base and BigBirdPegasus-large attention shapes, d = 64,
block = 64, r = 3, at 1K to 32K tokens, and the BigBird-base shape at block 128
and at d = 128):

=====================  ==========================  =========================================
name                   shape                       values / padding
=====================  ==========================  =========================================
tiny_l1024             B1 H2 L1024 (16 blocks)     N(0,1) fp32 -> bf16, no padding
bigbird_base_l4096     B4 H12 L4096                N(0,1)/sqrt(d); valid length U[2048, 4096]
pegasus_large_l4096    B2 H16 L4096                N(0,1); no padding
long_l16384            B1 H12 L16384 (256 blocks)  N(0,1); last 10 % of tokens padded
extreme_l32768         B1 H8 L32768 (512 blocks)   N(0,1) x 2; valid length U[24576, 32768]
base_l4096_block128    B4 H12 L4096, block 128     N(0,1)/sqrt(d); valid length U[2048, 4096]
base_l4096_d128        B4 H12 L4096, d 128         N(0,1)/sqrt(d); valid length U[2048, 4096]
=====================  ==========================  =========================================

Recipe: a ``torch.Generator`` seeded with the workload seed draws fp32 N(0,1)
for Q, then K, then V (each [B, H, L, d]), scales them, and rounds to bf16
(round-to-nearest-even, ``Tensor.to(torch.bfloat16)``). Valid lengths are then
drawn from the same generator (``torch.randint`` over the inclusive range).
Padding is on the right: token t of sequence b is valid iff t < valid_len[b].
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int = 64
    block: int = 64
    r: int = 3
    value_scale: float = 1.0
    pad: tuple | None = None  # None | ("uniform", lo, hi) | ("last_frac", f)
    seed: int = 0

    @property
    def nb(self) -> int:
        return self.L // self.block

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny_l1024", 1, 2, 1024, seed=1001),
        Workload("bigbird_base_l4096", 4, 12, 4096, value_scale=1.0 / math.sqrt(64.0),
                 pad=("uniform", 2048, 4096), seed=1002),
        Workload("pegasus_large_l4096", 2, 16, 4096, seed=1003),
        Workload("long_l16384", 1, 12, 16384, pad=("last_frac", 0.1), seed=1004),
        Workload("extreme_l32768", 1, 8, 32768, value_scale=2.0,
                 pad=("uniform", 24576, 32768), seed=1005),
        # the BigBird-base shape at the other sizes the pages allow (CUDA-core kernel)
        Workload("base_l4096_block128", 4, 12, 4096, block=128, value_scale=1.0 / math.sqrt(64.0),
                 pad=("uniform", 2048, 4096), seed=1006),
        Workload("base_l4096_d128", 4, 12, 4096, d=128, value_scale=1.0 / math.sqrt(128.0),
                 pad=("uniform", 2048, 4096), seed=1007),
    )
}


def valid_lengths(w: Workload, gen: torch.Generator) -> list[int]:
    """Per-sequence valid lengths (right padding)."""
    if w.pad is None:
        return [w.L] * w.B
    kind = w.pad[0]
    if kind == "uniform":
        lo, hi = int(w.pad[1]), int(w.pad[2])
        return [int(x) for x in torch.randint(lo, hi + 1, (w.B,), generator=gen)]
    if kind == "last_frac":
        return [w.L - int(math.floor(float(w.pad[1]) * w.L))] * w.B
    if kind == "fixed":
        return [int(x) for x in w.pad[1]]
    raise ValueError(f"unknown padding kind {kind!r}")


def make_inputs(w: Workload, seed: int | None = None) -> dict:
    """Draw one batch on the CPU: q, k, v (bf16 [B, H, L, d]), seq_mask (uint8
    [B, L], 1 = valid) or None when nothing is padded, and valid_len."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    shape = (w.B, w.H, w.L, w.d)
    q = (torch.randn(shape, generator=gen) * w.value_scale).to(torch.bfloat16)
    k = (torch.randn(shape, generator=gen) * w.value_scale).to(torch.bfloat16)
    v = (torch.randn(shape, generator=gen) * w.value_scale).to(torch.bfloat16)
    vl = valid_lengths(w, gen)
    if w.pad is None:
        seq_mask = None
    else:
        pos = torch.arange(w.L)
        seq_mask = torch.stack([(pos < n).to(torch.uint8) for n in vl])
    return {"q": q, "k": k, "v": v, "seq_mask": seq_mask, "valid_len": vl}


def mask_from_lengths(B: int, L: int, valid_len) -> torch.Tensor:
    """uint8 [B, L] right-padding mask from valid lengths."""
    pos = torch.arange(L)
    return torch.stack([(pos < int(n)).to(torch.uint8) for n in valid_len[:B]])
