"""BigBird ITC block-sparse attention on B200 (sm_100a): forward (fwd,
fwd_train), backward (bwd) and the attention-probability export (probs,
probs_dense).

Thin Python binding over the C ABI of ``libbigbird_attn.so`` (declared in
``include/bigbird_attn.h``): argument marshalling only. Every step runs in
the library's CUDA kernels; PyTorch supplies device memory and the current
stream. There is no CPU fallback: if the library is missing or no sm_100
device is present the calls raise.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbigbird_attn.so")

BB_OK, BB_ERR_INVALID_ARG, BB_ERR_UNSUPPORTED, BB_ERR_CUDA, BB_ERR_BAD_RAND_ATTN, BB_ERR_DEVICE = range(6)
BB_OUT_BF16, BB_OUT_F32 = 0, 1
BB_FLAG_FORCE_SPARSE, BB_FLAG_DEBUG_CHECKS = 1, 2

_lib = None


class BigBirdError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m block_sparse_long_attention_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, U, Z, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t, ctypes.c_uint64
    sig = {
        "bigbird_attn_fwd": (I, [P, P, P, P, P, P, I, I, I, I, I, I, P]),
        "bigbird_attn_fwd_ex": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I, U, P, Z, P]),
        "bigbird_attn_workspace_size": (Z, [I, I, I, I, I, I, U]),
        "bigbird_attn_is_fallback": (I, [I, I, I]),
        "bigbird_rand_attn_generate": (I, [P, I, I, I, I, U64, I]),
        "bigbird_rand_attn_validate": (I, [P, I, I, I, I, I]),
        "bigbird_mask_prep": (I, [P, I, I, I, P, P, P, P]),
        "bigbird_pattern_table": (I, [P, I, I, I, I, P]),
        "bigbird_device_status": (I, [P, ctypes.POINTER(ctypes.c_uint32)]),
        "bigbird_status_string": (ctypes.c_char_p, [I]),
        "bigbird_attn_fwd_noalloc": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I, U, P]),
        "bigbird_attn_noalloc_scratch_bytes": (Z, []),
        "bigbird_attn_fwd_train": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, U, P, Z, P]),
        "bigbird_attn_bwd": (I, [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, U, P]),
        "bigbird_attn_bwd_ex": (I, [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, U, P, Z, P]),
        "bigbird_attn_bwd_workspace_size": (Z, [I, I, I, I, I, I, U]),
        "bigbird_attn_fwd_host": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I, U, P, Z, P]),
        "bigbird_attn_fwd_host_scratch_bytes": (Z, [I, I, I, I, I, I, U]),
        "bigbird_wait_probe": (I, [U, P]),
        "bigbird_attn_probs_layout": (I, [I, I, I, I, U, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I)]),
        "bigbird_attn_probs": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, U, P]),
        "bigbird_attn_probs_dense": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I, U, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def lib():
    """The loaded ctypes library (raises ImportError if it is not built)."""
    return _load()


def status_string(status: int) -> str:
    return _load().bigbird_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != BB_OK:
        raise BigBirdError(status, what)


def _np_ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


# ------------------------------------------------------------------ host prep

def is_fallback(L: int, block: int = 64, r: int = 3) -> bool:
    res = _load().bigbird_attn_is_fallback(L, block, r)
    if res < 0:
        raise BigBirdError(BB_ERR_INVALID_ARG, "is_fallback")
    return bool(res)


def rand_attn_generate(H: int, L: int, block: int = 64, r: int = 3, seed: int = 0, last_idx: int = 0) -> np.ndarray:
    """Seeded random adjacency int32 [H, nb-2, r] (host)."""
    nb = L // block if block > 0 else 0
    out = np.empty((H, max(nb - 2, 0), r), dtype=np.int32)
    _check(_load().bigbird_rand_attn_generate(_np_ptr(out), H, L, block, r, seed & (2**64 - 1), last_idx),
           "rand_attn_generate")
    return out


def rand_attn_validate(rand_attn, H: int, L: int, block: int = 64, r: int = 3, last_idx: int = 0) -> int:
    """Status of the generator-rule check of a host rand_attn (BB_OK or an error code)."""
    ra = np.ascontiguousarray(rand_attn, dtype=np.int32)
    nb = L // block
    if ra.shape != (H, nb - 2, r):
        return BB_ERR_INVALID_ARG
    return _load().bigbird_rand_attn_validate(_np_ptr(ra), H, L, block, r, last_idx)


def mask_prep(seq_mask, block: int = 64):
    """(blocked [B,nb,bs], band [B,nb-4,bs,3bs], from_mask [B,L], to_mask [B,L]) uint8."""
    m = np.ascontiguousarray(np.asarray(seq_mask), dtype=np.uint8)
    B, L = m.shape
    nb = L // block
    blocked = np.empty((B, nb, block), np.uint8)
    band = np.empty((B, max(nb - 4, 0), block, 3 * block), np.uint8)
    frm = np.empty((B, L), np.uint8)
    to = np.empty((B, L), np.uint8)
    _check(_load().bigbird_mask_prep(_np_ptr(m), B, L, block, _np_ptr(blocked), _np_ptr(band), _np_ptr(frm),
                                     _np_ptr(to)), "mask_prep")
    return blocked, band, frm, to


def pattern_table(rand_attn, H: int, L: int, block: int = 64, r: int = 3) -> np.ndarray:
    """Sorted distinct key blocks per non-global query block: int32 [H, nb-2, 5+r], -1 padded."""
    ra = np.ascontiguousarray(rand_attn, dtype=np.int32)
    nb = L // block
    out = np.empty((H, nb - 2, 5 + r), np.int32)
    _check(_load().bigbird_pattern_table(_np_ptr(ra), H, L, block, r, _np_ptr(out)), "pattern_table")
    return out


# ------------------------------------------------------------------ forward

def workspace_size(B: int, H: int, L: int, d: int = 64, block: int = 64, r: int = 3, force_sparse: bool = False) -> int:
    flags = BB_FLAG_FORCE_SPARSE if force_sparse else 0
    return int(_load().bigbird_attn_workspace_size(B, H, L, d, block, r, flags))


def _stream_handle(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_inputs(q, k, v, rand_attn, seq_mask, block, r):
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 4):
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [B, H, L, d]")
    B, H, L, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v shapes differ")
    ra_ptr = None
    if rand_attn is not None:
        if not (rand_attn.is_cuda and rand_attn.dtype == torch.int32 and rand_attn.is_contiguous()):
            raise ValueError("rand_attn must be a contiguous int32 CUDA tensor [H, nb-2, r]")
        if rand_attn.shape != (H, L // block - 2, r):
            raise ValueError(f"rand_attn shape {tuple(rand_attn.shape)} != {(H, L // block - 2, r)}")
        ra_ptr = rand_attn.data_ptr()
    sm_ptr = None
    if seq_mask is not None:
        if not (seq_mask.is_cuda and seq_mask.dtype == torch.uint8 and seq_mask.is_contiguous()
                and seq_mask.shape == (B, L)):
            raise ValueError("seq_mask must be a contiguous uint8 CUDA tensor [B, L]")
        sm_ptr = seq_mask.data_ptr()
    return B, H, L, d, ra_ptr, sm_ptr


def fwd_train(q, k, v, rand_attn, seq_mask=None, *, block: int = 64, r: int = 3, out_dtype=None,
              force_sparse: bool = False, workspace=None, stream=None):
    """Forward for training: returns (out, lse) with lse [B, H, L] fp32 the
    natural-log log-sum-exp of each row's scores (what bwd() needs)."""
    import torch
    B, H, L, d, ra_ptr, sm_ptr = _check_inputs(q, k, v, rand_attn, seq_mask, block, r)
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bf16 or fp32")
    out = torch.empty((B, H, L, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    flags = BB_FLAG_FORCE_SPARSE if force_sparse else 0
    lib_ = _load()
    ws_bytes = int(lib_.bigbird_attn_workspace_size(B, H, L, d, block, r, flags))
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.zeros(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    st = lib_.bigbird_attn_fwd_train(q.data_ptr(), k.data_ptr(), v.data_ptr(), ra_ptr, sm_ptr, out.data_ptr(),
                                     lse.data_ptr(), B, H, L, d, block, r,
                                     BB_OUT_F32 if out_dtype == torch.float32 else BB_OUT_BF16, flags,
                                     workspace.data_ptr(), ws_bytes, _stream_handle(stream))
    _check(st, "bigbird_attn_fwd_train")
    return out, lse


def fwd_host_scratch_bytes(B: int, H: int, L: int, d: int = 64, block: int = 64, r: int = 3,
                           force_sparse: bool = False) -> int:
    flags = BB_FLAG_FORCE_SPARSE if force_sparse else 0
    return int(_load().bigbird_attn_fwd_host_scratch_bytes(B, H, L, d, block, r, flags))


def fwd_host(q, k, v, rand_attn, seq_mask, out, *, block: int = 64, r: int = 3, scratch=None,
             force_sparse: bool = False, stream=None):
    """bigbird_attn_fwd_host: q, k, v (bf16 [B, H, L, d]), rand_attn (int32
    [H, nb-2, r] or None), seq_mask (uint8 [B, L] or None) and out (bf16 or
    fp32, q's shape) are CPU tensors, page-locked for the copies to overlap
    compute; scratch a uint8 CUDA tensor of fwd_host_scratch_bytes(...) bytes.
    Runs on the current torch stream (or `stream`); synchronise it before
    reading out."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor [B, H, L, d]")
    if k.shape != q.shape or v.shape != q.shape or out.shape != q.shape or out.is_cuda or not out.is_contiguous():
        raise ValueError("k, v and out must be contiguous CPU tensors of q's shape")
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bf16 or fp32")
    B, H, L, d = q.shape
    flags = BB_FLAG_FORCE_SPARSE if force_sparse else 0
    need = fwd_host_scratch_bytes(B, H, L, d, block, r, force_sparse)
    if scratch is None or not scratch.is_cuda or scratch.numel() * scratch.element_size() < need:
        raise ValueError(f"scratch must be a CUDA tensor of at least {need} bytes")
    ra = None
    if rand_attn is not None:
        ra = torch.as_tensor(rand_attn, dtype=torch.int32).contiguous()
        if ra.is_cuda:
            raise ValueError("rand_attn must be on the host")
    if seq_mask is not None and (seq_mask.is_cuda or seq_mask.dtype != torch.uint8 or not seq_mask.is_contiguous()):
        raise ValueError("seq_mask must be a contiguous uint8 CPU tensor [B, L]")
    st = _load().bigbird_attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       None if ra is None else ra.data_ptr(),
                                       None if seq_mask is None else seq_mask.data_ptr(), out.data_ptr(),
                                       B, H, L, d, block, r, BB_OUT_F32 if out.dtype == torch.float32 else BB_OUT_BF16,
                                       flags, scratch.data_ptr(), need, _stream_handle(stream))
    _check(st, "bigbird_attn_fwd_host")
    return out


def bwd_workspace_size(B: int, H: int, L: int, d: int = 64, block: int = 64, r: int = 3,
                       force_sparse: bool = False) -> int:
    flags = BB_FLAG_FORCE_SPARSE if force_sparse else 0
    return int(_load().bigbird_attn_bwd_workspace_size(B, H, L, d, block, r, flags))


def bwd(q, k, v, out, dout, lse, rand_attn, seq_mask=None, *, block: int = 64, r: int = 3,
        force_sparse: bool = False, stream=None, workspace=None):
    """Backward: returns (dq, dk, dv), fp32 [B, H, L, d], the gradients of
    sum(dout * out). out is the forward's output (bf16 or fp32), dout a bf16
    tensor of its shape, lse from fwd_train(). `workspace` (optional, reusable
    across calls): a uint8 CUDA tensor of at least bwd_workspace_size(...)
    bytes, zero-filled before its first use (e.g. torch.zeros)."""
    import torch
    B, H, L, d, ra_ptr, sm_ptr = _check_inputs(q, k, v, rand_attn, seq_mask, block, r)
    if not (dout.is_cuda and dout.dtype == torch.bfloat16 and dout.is_contiguous() and dout.shape == q.shape):
        raise ValueError("dout must be a contiguous bf16 CUDA tensor of q's shape")
    if not (out.is_cuda and out.dtype in (torch.bfloat16, torch.float32) and out.is_contiguous()
            and out.shape == q.shape):
        raise ValueError("out must be the forward's output (bf16 or fp32, q's shape)")
    if not (lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and lse.shape == (B, H, L)):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, H, L]")
    dq, dk, dv = (torch.empty((B, H, L, d), dtype=torch.float32, device=q.device) for _ in range(3))
    flags = BB_FLAG_FORCE_SPARSE if force_sparse else 0
    lib_ = _load()
    ws_bytes = int(lib_.bigbird_attn_bwd_workspace_size(B, H, L, d, block, r, flags))
    ws_ptr = None
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < ws_bytes:
            raise ValueError(f"workspace too small: need {ws_bytes} bytes")
        ws_ptr = workspace.data_ptr()
    st = lib_.bigbird_attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                                  lse.data_ptr(), ra_ptr, sm_ptr, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                  B, H, L, d, block, r, BB_OUT_F32 if out.dtype == torch.float32 else BB_OUT_BF16,
                                  flags, ws_ptr, ws_bytes if ws_ptr else 0, _stream_handle(stream))
    _check(st, "bigbird_attn_bwd_ex")
    return dq, dk, dv


def probs_layout(L: int, block: int = 64, r: int = 3, d: int = 64, force_sparse: bool = False):
    """(G, band_rows, band_slots) of the packed probability layout: G full
    rows per head (2 sparse, nb in the fallback), band tiles
    [nb-2, 5+r] per head (0, 0 in the fallback)."""
    g, br, bs = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    st = _load().bigbird_attn_probs_layout(L, d, block, r, BB_FLAG_FORCE_SPARSE if force_sparse else 0,
                                          ctypes.byref(g), ctypes.byref(br), ctypes.byref(bs))
    _check(st, "bigbird_attn_probs_layout")
    return g.value, br.value, bs.value


def _probs_args(q, k, lse, rand_attn, seq_mask, block, r, out_dtype):
    import torch
    B, H, L, d, ra_ptr, sm_ptr = _check_inputs(q, k, k, rand_attn, seq_mask, block, r)
    if not (lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and lse.shape == (B, H, L)):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, H, L] (from fwd_train)")
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bf16 or fp32")
    return B, H, L, d, ra_ptr, sm_ptr, out_dtype


def probs(q, k, lse, rand_attn, seq_mask=None, *, block: int = 64, r: int = 3, out_dtype=None,
          force_sparse: bool = False, out=None, stream=None):
    """Attention weights in the packed block-sparse layout: returns
    (probs_global [B, H, G, 64, L], probs_band [B, H, nb-2, 5+r, 64, 64] or
    None in the fallback). Tile t of band row i is against key block
    pattern_table(...)[h, i-1, t] (zeros where that entry is -1). lse comes
    from fwd_train() on the same inputs. Default dtype fp32. `out` may be a
    (probs_global, probs_band) pair of preallocated contiguous tensors."""
    import torch
    B, H, L, d, ra_ptr, sm_ptr, out_dtype = _probs_args(q, k, lse, rand_attn, seq_mask, block, r, out_dtype)
    G, nbr, slots = probs_layout(L, block, r, d, force_sparse)
    shapes = ((B, H, G, block, L), (B, H, nbr, slots, block, block) if nbr else None)
    if out is None:
        pg = torch.empty(shapes[0], dtype=out_dtype, device=q.device)
        pb = torch.empty(shapes[1], dtype=out_dtype, device=q.device) if nbr else None
    else:
        pg, pb = out
        for t, shp in ((pg, shapes[0]), (pb, shapes[1])):
            if shp is None:
                continue
            if t is None or not (t.is_cuda and t.dtype == out_dtype and t.is_contiguous() and tuple(t.shape) == shp):
                raise ValueError(f"out tensors must be contiguous CUDA tensors {shapes} of {out_dtype}")
    st = _load().bigbird_attn_probs(q.data_ptr(), k.data_ptr(), lse.data_ptr(), ra_ptr, sm_ptr, pg.data_ptr(),
                                    None if pb is None else pb.data_ptr(), B, H, L, d, block, r,
                                    BB_OUT_F32 if out_dtype == torch.float32 else BB_OUT_BF16,
                                    BB_FLAG_FORCE_SPARSE if force_sparse else 0, _stream_handle(stream))
    _check(st, "bigbird_attn_probs")
    return pg, pb


def probs_dense(q, k, lse, rand_attn, seq_mask=None, *, block: int = 64, r: int = 3, out_dtype=None,
                force_sparse: bool = False, out=None, stream=None):
    """Attention weights as the full [B, H, L, L] matrix (zeros outside the
    pattern), the layout the model returns for its attention outputs."""
    import torch
    B, H, L, d, ra_ptr, sm_ptr, out_dtype = _probs_args(q, k, lse, rand_attn, seq_mask, block, r, out_dtype)
    if out is None:
        out = torch.empty((B, H, L, L), dtype=out_dtype, device=q.device)
    elif not (out.is_cuda and out.dtype == out_dtype and out.is_contiguous() and out.shape == (B, H, L, L)):
        raise ValueError("out must be a contiguous CUDA tensor [B, H, L, L] of out_dtype")
    st = _load().bigbird_attn_probs_dense(q.data_ptr(), k.data_ptr(), lse.data_ptr(), ra_ptr, sm_ptr,
                                          out.data_ptr(), B, H, L, d, block, r,
                                          BB_OUT_F32 if out_dtype == torch.float32 else BB_OUT_BF16,
                                          BB_FLAG_FORCE_SPARSE if force_sparse else 0, _stream_handle(stream))
    _check(st, "bigbird_attn_probs_dense")
    return out


def fwd(q, k, v, rand_attn, seq_mask=None, *, block: int = 64, r: int = 3, out=None, out_dtype=None,
        force_sparse: bool = False, debug_checks: bool = False, workspace=None, stream=None):
    """BigBird ITC attention forward: returns out [B, H, L, d] (bf16, or fp32
    with out_dtype=torch.float32). q, k, v: contiguous bf16 CUDA tensors
    [B, H, L, d]; rand_attn: int32 CUDA tensor [H, nb-2, r] (or None in the
    full-attention fallback); seq_mask: uint8 CUDA tensor [B, L] (1 = valid
    key) or None. Runs on the current torch stream (or `stream`).
    `workspace` (optional, reusable across calls): a uint8 CUDA tensor of at
    least workspace_size(...) bytes, zero-filled before its first use (each
    call leaves its counters at zero again, e.g. torch.zeros)."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 4):
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [B, H, L, d]")
    B, H, L, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v shapes differ")
    if out_dtype is None:
        out_dtype = torch.bfloat16 if out is None else out.dtype
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bf16 or fp32")
    if out is None:
        out = torch.empty((B, H, L, d), dtype=out_dtype, device=q.device)
    elif not (out.is_cuda and out.dtype == out_dtype and out.is_contiguous() and out.shape == q.shape):
        raise ValueError("out must be a contiguous CUDA tensor of q's shape and out_dtype")
    ra_ptr = None
    if rand_attn is not None:
        if not (rand_attn.is_cuda and rand_attn.dtype == torch.int32 and rand_attn.is_contiguous()):
            raise ValueError("rand_attn must be a contiguous int32 CUDA tensor [H, nb-2, r]")
        if rand_attn.shape != (H, L // block - 2, r):
            raise ValueError(f"rand_attn shape {tuple(rand_attn.shape)} != {(H, L // block - 2, r)}")
        ra_ptr = rand_attn.data_ptr()
    sm_ptr = None
    if seq_mask is not None:
        if not (seq_mask.is_cuda and seq_mask.dtype == torch.uint8 and seq_mask.is_contiguous()
                and seq_mask.shape == (B, L)):
            raise ValueError("seq_mask must be a contiguous uint8 CUDA tensor [B, L]")
        sm_ptr = seq_mask.data_ptr()
    flags = (BB_FLAG_FORCE_SPARSE if force_sparse else 0) | (BB_FLAG_DEBUG_CHECKS if debug_checks else 0)
    lib_ = _load()
    ws_bytes = int(lib_.bigbird_attn_workspace_size(B, H, L, d, block, r, flags))
    ws_ptr = None
    if ws_bytes:
        if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
            workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=q.device)
        ws_ptr = workspace.data_ptr()
    st = lib_.bigbird_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), ra_ptr, sm_ptr, out.data_ptr(),
                                  B, H, L, d, block, r, BB_OUT_F32 if out_dtype == torch.float32 else BB_OUT_BF16,
                                  flags, ws_ptr, ws_bytes, _stream_handle(stream))
    _check(st, "bigbird_attn_fwd_ex")
    return out


def device_status(stream=None) -> int:
    """Synchronise the stream, then read and clear the device error word
    (bit 1: out-of-range rand_attn entry skipped; bit 2: a kernel wait timed out)."""
    v = ctypes.c_uint32(0)
    _check(_load().bigbird_device_status(_stream_handle(stream), ctypes.byref(v)), "device_status")
    return int(v.value)


__all__ = [
    "BigBirdError", "fwd", "fwd_train", "bwd", "probs", "probs_dense", "probs_layout", "workspace_size", "is_fallback", "rand_attn_generate", "rand_attn_validate",
    "mask_prep", "pattern_table", "device_status", "status_string", "lib", "LIB_PATH",
]
