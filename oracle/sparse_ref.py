"""ctypes wrapper of sparse_ref.c: the sparse brute-force CPU reference.

TEST AND BENCHMARK INFRASTRUCTURE ONLY (see the package docstring). The C
code computes the same definition as ``attention`` but visits only each row's
keys, in fp64, with OpenMP threads; the tests pin it against ``attention`` and
``bench.py`` times it as the fair CPU baseline.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sparse_ref.c")
LIB = os.path.join(HERE, "libbigbird_sparse_ref.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile sparse_ref.c with gcc -O2 -fopenmp into oracle/ (in-tree)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", LIB, SRC, "-lm"], check=True)
    return LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        lib.bigbird_sparse_ref.argtypes = [P, P, P, P, P, P] + [ctypes.c_int] * 8
        lib.bigbird_sparse_ref.restype = ctypes.c_int
        _lib = lib
    return _lib


def _bf16_bits(x) -> np.ndarray:
    """bf16 bit patterns of a torch bf16 tensor (or of float values rounded to bf16)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.to(torch.bfloat16).contiguous().view(torch.int16).numpy()).view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    bits = a.view(np.uint32)
    rounded = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16  # round to nearest even
    return rounded.astype(np.uint16)


def sparse_attention(q, k, v, rand_attn, seq_mask, block: int, r: int, force_sparse: bool = False,
                     threads: int | None = None) -> np.ndarray:
    """out[B, H, L, d] in fp64 from the C sparse reference (inputs used at their bf16 values)."""
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    B, H, L, d = qb.shape
    ra = None if rand_attn is None else np.ascontiguousarray(np.asarray(rand_attn, dtype=np.int32))
    sm = None if seq_mask is None else np.ascontiguousarray(np.asarray(seq_mask).astype(np.uint8))
    out = np.empty((B, H, L, d), dtype=np.float64)
    n = threads or len(os.sched_getaffinity(0))
    st = _load().bigbird_sparse_ref(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data,
                                    None if ra is None else ra.ctypes.data, None if sm is None else sm.ctypes.data,
                                    out.ctypes.data, B, H, L, d, block, r, int(force_sparse), n)
    if st != 0:
        raise ValueError(f"sparse reference: status {st}")
    return out
