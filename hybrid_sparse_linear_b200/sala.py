"""ctypes binding of libsala (``include/sala.h``).

Argument marshalling only: every function checks that the torch tensors it is given have the
layout the C ABI documents, then passes raw device pointers and the current CUDA stream.  All
computation happens in the library's CUDA kernels; there is no CPU or PyTorch fallback -- if the
library is missing this module fails to import.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SALA_LIBRARY=debug loads the bounds-checking build (libsala_debug.so: the same kernels, with
# out-of-range indices recorded as SALA_ERR_BOUNDS and skipped); anything else the release build.
LIB_PATH = os.path.join(_HERE, "libsala_debug.so" if os.environ.get("SALA_LIBRARY") == "debug"
                        else "libsala.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m hybrid_sparse_linear_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = range(6)
F32, BF16 = 0, 1

_vp, _i, _st = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_lib.sala_linear_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
_lib.sala_linear_prefill_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp,
                                        ctypes.c_size_t, _i, _vp]
_lib.sala_linear_prefill_workspace.argtypes = [_i, _i, _i, _i, _i]
_lib.sala_linear_prefill_workspace.restype = ctypes.c_size_t
_lib.sala_linear_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]
_lib.sala_linear_backward.argtypes = [_vp] * 8 + [_i] * 4 + [_vp, _st, _i, _vp]
_lib.sala_linear_backward_workspace.argtypes = [_i] * 5
_lib.sala_linear_backward_workspace.restype = _st
_lib.sala_linear_prefill_rope.argtypes = [_vp] * 7 + [_i] * 4 + [ctypes.c_int64, ctypes.c_double,
                                                              _vp, _st, _i, _vp]
_lib.sala_linear_decode_rope.argtypes = [_vp] * 6 + [_i] * 3 + [ctypes.c_int64, ctypes.c_double, _i, _vp]
_lib.sala_linear_decode_pdl.argtypes = [_vp] * 6 + [_i] * 3 + [ctypes.c_int64, ctypes.c_double, _i, _vp]
_lib.sala_qk_norm.argtypes = [_vp, _vp, ctypes.c_int64, _vp, _vp, ctypes.c_int64, _i,
                              ctypes.c_double, _i, _vp]
_lib.sala_qk_prologue.argtypes = [_vp, _vp, ctypes.c_int64, _vp, _vp, ctypes.c_int64, _i, _i,
                                  ctypes.c_double, ctypes.c_int64, ctypes.c_double, _i, _vp]
_lib.sala_block_compress.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp]
_lib.sala_block_topk.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                                 _st, _i, _vp]
_lib.sala_block_topk_workspace.argtypes = [_i, _i, _i, _i, _i, _i, _i]
_lib.sala_block_topk_qblock.argtypes = [_vp, _vp, _vp] + [_i] * 11 + [_vp]
_lib.sala_block_topk_qblock_softmax.argtypes = [_vp, _vp, _vp] + [_i] * 10 + [ctypes.c_float, _i, _vp]
_lib.sala_block_topk_per_head.argtypes = [_vp, _vp, _vp] + [_i] * 11 + [_vp]
_lib.sala_block_topk_workspace.restype = _st
_lib.sala_sparse_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                     ctypes.c_float, _i, _vp]
_lib.sala_sparse_prefill_per_head.argtypes = _lib.sala_sparse_prefill.argtypes
_lib.sala_sparse_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                    _i, _i, _i, _i, ctypes.c_float, _vp, _st, _i, _vp]
_lib.sala_sparse_decode_pdl.argtypes = _lib.sala_sparse_decode.argtypes
_lib.sala_sparse_decode_workspace.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i, _i]
_lib.sala_sparse_decode_workspace.restype = _st
_lib.sala_sparse_decode_paged.argtypes = [_vp, _vp, _vp, _i, _vp, _i, _vp, _i, _vp, _i, _vp, _vp,
                                          _i, _i, _i, _i, _i, _i, _i, _i, ctypes.c_float, _vp, _st,
                                          _i, _vp]
_lib.sala_sparse_decode_paged_workspace.argtypes = [_i] * 9
_lib.sala_sparse_decode_paged_workspace.restype = _st
_lib.sala_sparse_prefill_lse.argtypes = [_vp] * 7 + [_i] * 7 + [ctypes.c_float, _i, _vp]
_lib.sala_sparse_backward_workspace.argtypes = [_i] * 6
_lib.sala_sparse_backward_workspace.restype = _st
_lib.sala_sparse_backward.argtypes = [_vp] * 11 + [_i] * 7 + [ctypes.c_float, _vp, _st, _i, _vp]
_lib.sala_check_status.argtypes = [_vp]
_lib.sala_debug_bounds_build.restype = _i
_lib.sala_status_string.argtypes = [_i]
_lib.sala_status_string.restype = ctypes.c_char_p
_lib.sala_last_error.restype = ctypes.c_char_p
_lib.sala_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.sala_selftest_wait_timeout.argtypes = [_vp]
for _f in ("sala_linear_prefill", "sala_linear_decode", "sala_linear_prefill_rope",
           "sala_linear_decode_rope", "sala_sparse_decode_paged", "sala_block_topk_qblock",
           "sala_linear_backward", "sala_qk_norm", "sala_sparse_prefill_lse", "sala_sparse_backward",
           "sala_block_topk_qblock_softmax", "sala_linear_decode_pdl", "sala_qk_prologue",
           "sala_block_topk_per_head", "sala_sparse_prefill_per_head",
           "sala_block_compress",
           "sala_block_topk",
           "sala_sparse_prefill", "sala_sparse_decode", "sala_sparse_decode_pdl", "sala_check_status",
           "sala_selftest_wait_timeout"):
    getattr(_lib, _f).restype = _i


class SalaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = _lib.sala_last_error().decode()
        super().__init__(f"{where}: {_lib.sala_status_string(code).decode()}: {msg}")


def _check(code: int, where: str):
    if code != OK:
        raise SalaError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _need(t, name, shape=None, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


# ----------------------------------------------------------------------------------------------
def linear_prefill_workspace_bytes(B, H, N, d, dtype=torch.bfloat16):
    return _lib.sala_linear_prefill_workspace(B, H, N, d, 1 if dtype == torch.bfloat16 else 0)


def linear_prefill(q, k, v, decay, o=None, state_in=None, state_out=None, chunk=0, workspace=None,
                   stream=None, rope_base=None, pos0=0):
    """Chunked decayed linear attention.  q,k,v: [B,H,N,d]; decay [H] fp32.  Returns o.
    workspace: None = one pass (sala_linear_prefill); a uint8 device tensor of at least
    linear_prefill_workspace_bytes(...) bytes lets long sequences run as parallel segments
    (sala_linear_prefill_ws).  rope_base: rotate q and k by position first, row r at pos0 + r
    (sala_linear_prefill_rope; chunk is then the kernel's own)."""
    B, H, N, d = q.shape
    _need(q, "q"); _need(k, "k", q.shape, q.dtype); _need(v, "v", q.shape, q.dtype)
    _need(decay, "decay", (H,), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype)
    _need(state_in, "state_in", (B, H, d, d), torch.float32)
    _need(state_out, "state_out", (B, H, d, d), torch.float32)
    if rope_base is not None:
        _check(_lib.sala_linear_prefill_rope(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(o),
                                             _ptr(state_in), _ptr(state_out), B, H, N, d, int(pos0),
                                             float(rope_base), _ptr(workspace),
                                             0 if workspace is None else workspace.numel(), _dt(q),
                                             _stream(stream)), "sala_linear_prefill_rope")
    elif workspace is None:
        _check(_lib.sala_linear_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(o),
                                        _ptr(state_in), _ptr(state_out), B, H, N, d, chunk, _dt(q),
                                        _stream(stream)), "sala_linear_prefill")
    else:
        _check(_lib.sala_linear_prefill_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(o),
                                           _ptr(state_in), _ptr(state_out), B, H, N, d, chunk,
                                           _ptr(workspace), workspace.numel(), _dt(q),
                                           _stream(stream)), "sala_linear_prefill_ws")
    return o


def linear_backward(q, k, v, decay, dout, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of sum(o * dout) for the linear attention of a fresh sequence.
    q, k, v, dout: [B,H,N,d]; decay [H] fp32."""
    B, H, N, d = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _need(t, n, q.shape, q.dtype)
    _need(decay, "decay", (H,), torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    need = _lib.sala_linear_backward_workspace(B, H, N, d, _dt(q))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(_lib.sala_linear_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(dout), _ptr(dq),
                                     _ptr(dk), _ptr(dv), B, H, N, d, _ptr(workspace),
                                     workspace.numel(), _dt(q), _stream(stream)),
           "sala_linear_backward")
    return dq, dk, dv


def linear_decode(q, k, v, decay, state, o=None, stream=None, rope_base=None, pos=0, pdl=False):
    """One decode step.  q,k,v: [B,H,d]; state [B,H,d,d] fp32 (updated in place).  Returns o.
    rope_base: rotate q and k at position pos first (sala_linear_decode_rope).  pdl: launch as a
    programmatic dependent of the previous kernel in the stream (sala_linear_decode_pdl; that
    kernel must not write `state`)."""
    B, H, d = q.shape
    _need(q, "q"); _need(k, "k", q.shape, q.dtype); _need(v, "v", q.shape, q.dtype)
    _need(decay, "decay", (H,), torch.float32)
    _need(state, "state", (B, H, d, d), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype)
    if pdl:
        _check(_lib.sala_linear_decode_pdl(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(state),
                                           _ptr(o), B, H, d, int(pos),
                                           float(rope_base) if rope_base is not None else 0.0,
                                           _dt(q), _stream(stream)), "sala_linear_decode_pdl")
        return o
    if rope_base is not None:
        _check(_lib.sala_linear_decode_rope(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(state),
                                            _ptr(o), B, H, d, int(pos), float(rope_base), _dt(q),
                                            _stream(stream)), "sala_linear_decode_rope")
        return o
    _check(_lib.sala_linear_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(state), _ptr(o),
                                   B, H, d, _dt(q), _stream(stream)), "sala_linear_decode")
    return o


def qk_norm(q, k=None, q_out=None, k_out=None, eps=1e-6, stream=None):
    """Weight-free RMS normalisation of every head row (last dim d) of q and, if given, k, in
    one launch.  Pass q_out=q / k_out=k to normalise in place.  Returns (q_out, k_out)."""
    d = q.shape[-1]
    _need(q, "q")
    if q_out is None:
        q_out = torch.empty_like(q)
    _need(q_out, "q_out", q.shape, q.dtype)
    k_rows = 0
    if k is not None:
        _need(k, "k", dtype=q.dtype)
        if k.shape[-1] != d:
            raise ValueError(f"k has head dim {k.shape[-1]}, q has {d}")
        if k_out is None:
            k_out = torch.empty_like(k)
        _need(k_out, "k_out", k.shape, k.dtype)
        k_rows = k.numel() // d
    _check(_lib.sala_qk_norm(_ptr(q), _ptr(q_out), q.numel() // d, _ptr(k), _ptr(k_out), k_rows,
                             d, float(eps), _dt(q), _stream(stream)), "sala_qk_norm")
    return q_out, k_out


def qk_prologue(q, k=None, q_out=None, k_out=None, eps=0.0, rope_base=0.0, pos0=0, stream=None):
    """One pass over q [B,H,N,d] and k [B,Hk,N,d]: the QK normalisation (eps > 0) and/or the
    linear layers' RoPE (rope_base > 0, row n at position pos0 + n).  Pass q_out=q / k_out=k to
    work in place.  Returns (q_out, k_out)."""
    N, d = q.shape[-2], q.shape[-1]
    _need(q, "q")
    if q_out is None:
        q_out = torch.empty_like(q)
    _need(q_out, "q_out", q.shape, q.dtype)
    k_rows = 0
    if k is not None:
        _need(k, "k", dtype=q.dtype)
        if k.shape[-2:] != q.shape[-2:]:
            raise ValueError(f"k has rows x dim {tuple(k.shape[-2:])}, q has {tuple(q.shape[-2:])}")
        if k_out is None:
            k_out = torch.empty_like(k)
        _need(k_out, "k_out", k.shape, k.dtype)
        k_rows = k.numel() // d
    _check(_lib.sala_qk_prologue(_ptr(q), _ptr(q_out), q.numel() // d, _ptr(k), _ptr(k_out), k_rows,
                                 d, N, float(eps), int(pos0), float(rope_base), _dt(q),
                                 _stream(stream)), "sala_qk_prologue")
    return q_out, k_out


def block_compress(k, kbar=None, block=64, first_block=0, n_blocks=None, stream=None):
    """Mean-pooled block keys.  k: [B,Hkv,N,d] -> kbar [B,Hkv,nb_cap,d]."""
    B, Hkv, N, d = k.shape
    _need(k, "k")
    if n_blocks is None:
        n_blocks = N // block - first_block
    if kbar is None:
        kbar = torch.empty((B, Hkv, first_block + n_blocks, d), device=k.device, dtype=k.dtype)
    _need(kbar, "kbar", dtype=k.dtype)
    _check(_lib.sala_block_compress(_ptr(k), _ptr(kbar), B, Hkv, N, d, block, first_block,
                                    n_blocks, kbar.shape[2], _dt(k), _stream(stream)),
           "sala_block_compress")
    return kbar


def block_topk(q, kbar, topk, n_init=1, n_local=1, block=64, q_pos0=0, idx=None, workspace=None,
               stream=None):
    """Per (batch, KV group, query row) block selection -> idx [B,Hkv,Nq,slots] int32."""
    B, H, Nq, d = q.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    _need(q, "q"); _need(kbar, "kbar", dtype=q.dtype)
    slots = n_init + n_local + topk
    if idx is None:
        idx = torch.empty((B, Hkv, Nq, slots), device=q.device, dtype=torch.int32)
    _need(idx, "idx", (B, Hkv, Nq, slots), torch.int32)
    need = _lib.sala_block_topk_workspace(B, Hkv, Nq, q_pos0, nb, block, topk)
    if need and workspace is None:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    _check(_lib.sala_block_topk(_ptr(q), _ptr(kbar), _ptr(idx), B, H, Hkv, Nq, q_pos0, nb, d,
                                block, topk, n_init, n_local, _ptr(workspace),
                                0 if workspace is None else workspace.numel(), _dt(q),
                                _stream(stream)), "sala_block_topk")
    return idx


def block_topk_qblock(q, kbar, topk, n_init, n_local, idx=None, block=64, stream=None):
    """Query-block-granular selection (one selection per KV group and query block, written to
    every token row).  q: [B,H,Nq,d]; kbar [B,Hkv,nb,d].  Returns idx [B,Hkv,Nq,slots] int32."""
    B, H, Nq, d = q.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    slots = n_init + n_local + topk
    _need(q, "q"); _need(kbar, "kbar", dtype=q.dtype)
    if idx is None:
        idx = torch.empty((B, Hkv, Nq, slots), dtype=torch.int32, device=q.device)
    _need(idx, "idx", (B, Hkv, Nq, slots), torch.int32)
    _check(_lib.sala_block_topk_qblock(_ptr(q), _ptr(kbar), _ptr(idx), B, H, Hkv, Nq, nb, d, block,
                                       topk, n_init, n_local, _dt(q), _stream(stream)),
           "sala_block_topk_qblock")
    return idx


def block_topk_qblock_softmax(q, kbar, topk, n_init, n_local, idx=None, block=64, scale=0.0,
                              stream=None):
    """Query-block-granular selection scored by softmax-probability group aggregation.
    q: [B,H,Nq,d]; kbar [B,Hkv,nb,d].  Returns idx [B,Hkv,Nq,slots] int32."""
    B, H, Nq, d = q.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    slots = n_init + n_local + topk
    _need(q, "q"); _need(kbar, "kbar", dtype=q.dtype)
    if idx is None:
        idx = torch.empty((B, Hkv, Nq, slots), dtype=torch.int32, device=q.device)
    _need(idx, "idx", (B, Hkv, Nq, slots), torch.int32)
    _check(_lib.sala_block_topk_qblock_softmax(_ptr(q), _ptr(kbar), _ptr(idx), B, H, Hkv, Nq, nb,
                                               d, block, topk, n_init, n_local, float(scale),
                                               _dt(q), _stream(stream)),
           "sala_block_topk_qblock_softmax")
    return idx


def block_topk_per_head(q, kbar, topk, n_init, n_local, idx=None, block=64, stream=None):
    """Per-query-head selection (each query head scores the candidates with its own query against
    its KV head's kbar).  q: [B,H,Nq,d]; kbar [B,Hkv,nb,d].  Returns idx [B,H,Nq,slots] int32."""
    B, H, Nq, d = q.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    slots = n_init + n_local + topk
    _need(q, "q"); _need(kbar, "kbar", dtype=q.dtype)
    if idx is None:
        idx = torch.empty((B, H, Nq, slots), dtype=torch.int32, device=q.device)
    _need(idx, "idx", (B, H, Nq, slots), torch.int32)
    _check(_lib.sala_block_topk_per_head(_ptr(q), _ptr(kbar), _ptr(idx), B, H, Hkv, Nq, nb, d,
                                         block, topk, n_init, n_local, _dt(q), _stream(stream)),
           "sala_block_topk_per_head")
    return idx


def sparse_prefill_per_head(q, k, v, idx, o=None, block=64, scale=0.0, stream=None):
    """Softmax attention over per-head selections.  q: [B,H,N,d]; k,v: [B,Hkv,N,d];
    idx [B,H,N,slots] int32 (block_topk_per_head's output)."""
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    _need(q, "q"); _need(k, "k", (B, Hkv, N, d), q.dtype); _need(v, "v", (B, Hkv, N, d), q.dtype)
    _need(idx, "idx", dtype=torch.int32)
    if idx.shape[:3] != (B, H, N):
        raise ValueError(f"idx has shape {tuple(idx.shape)}, expected ({B}, {H}, {N}, slots)")
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype)
    _check(_lib.sala_sparse_prefill_per_head(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o), B, H,
                                             Hkv, N, d, block, idx.shape[3], float(scale), _dt(q),
                                             _stream(stream)),
           "sala_sparse_prefill_per_head")
    return o


def sparse_prefill(q, k, v, idx, o=None, block=64, scale=0.0, stream=None, lse=None, o_lo=None):
    """Softmax attention over the selected blocks.  q: [B,H,N,d]; k,v: [B,Hkv,N,d].
    Training forward (sala_sparse_prefill_lse): lse = an fp32 [B,H,N] tensor, or True to allocate
    one, receives each row's log-sum-exp; o_lo (a tensor like q, or True to allocate; None for
    none) o's bf16 rounding residual.  Then (o, lse, o_lo) is returned."""
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    _need(q, "q"); _need(k, "k", (B, Hkv, N, d), q.dtype); _need(v, "v", (B, Hkv, N, d), q.dtype)
    _need(idx, "idx", dtype=torch.int32)
    if idx.shape[:3] != (B, Hkv, N):
        raise ValueError(f"idx has shape {tuple(idx.shape)}, expected ({B}, {Hkv}, {N}, slots)")
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype)
    if lse is not None:
        if lse is True:
            lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
        _need(lse, "lse", (B, H, N), torch.float32)
        if o_lo is True:
            o_lo = torch.empty_like(q)
        _need(o_lo, "o_lo", q.shape, q.dtype)
        _check(_lib.sala_sparse_prefill_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o), _ptr(lse),
                                            _ptr(o_lo), B, H, Hkv, N, d, block, idx.shape[3],
                                            float(scale), _dt(q), _stream(stream)),
               "sala_sparse_prefill_lse")
        return o, lse, o_lo
    _check(_lib.sala_sparse_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o), B, H, Hkv, N, d,
                                    block, idx.shape[3], float(scale), _dt(q), _stream(stream)),
           "sala_sparse_prefill")
    return o


def sparse_backward_workspace_bytes(B, H, Hkv, N, d, slots):
    return _lib.sala_sparse_backward_workspace(B, H, Hkv, N, d, slots)


def sparse_backward(q, k, v, idx, o, lse, dout, o_lo=None, block=64, scale=0.0, workspace=None,
                    stream=None):
    """Gradients (dq, dk, dv) of sum(o * dout) for the sparse attention with the selection idx
    held fixed.  o, lse, o_lo: from sparse_prefill(..., lse=True, o_lo=True)."""
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    _need(q, "q"); _need(k, "k", (B, Hkv, N, d), q.dtype); _need(v, "v", (B, Hkv, N, d), q.dtype)
    _need(o, "o", q.shape, q.dtype); _need(dout, "dout", q.shape, q.dtype)
    _need(o_lo, "o_lo", q.shape, q.dtype)
    _need(lse, "lse", (B, H, N), torch.float32)
    _need(idx, "idx", dtype=torch.int32)
    if idx.shape[:3] != (B, Hkv, N):
        raise ValueError(f"idx has shape {tuple(idx.shape)}, expected ({B}, {Hkv}, {N}, slots)")
    slots = idx.shape[3]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    need = _lib.sala_sparse_backward_workspace(B, H, Hkv, N, d, slots)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(_lib.sala_sparse_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o), _ptr(o_lo),
                                     _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, H, Hkv, N, d,
                                     block, slots, float(scale), _ptr(workspace),
                                     workspace.numel(), _dt(q), _stream(stream)),
           "sala_sparse_backward")
    return dq, dk, dv


def sparse_decode_workspace_bytes(B, H, Hkv, pos, topk, n_init, n_local, d, block=64):
    return _lib.sala_sparse_decode_workspace(B, H, Hkv, pos, block, topk, n_init, n_local, d)


def sparse_decode(q, kcache, vcache, kbar, pos, topk, n_init=1, n_local=2, idx_in=None,
                  idx_out=None, o=None, block=64, scale=0.0, workspace=None, stream=None, pdl=False):
    """One query token per head at position pos over a dense KV cache.  q: [B,H,d].
    pdl=True launches it as a programmatic dependent of the previous kernel in the stream
    (sala_sparse_decode_pdl: k_bar is read while that kernel finishes, so it must not write it)."""
    B, H, d = q.shape
    Hkv, Tmax = kcache.shape[1], kcache.shape[2]
    _need(q, "q"); _need(kcache, "kcache", dtype=q.dtype); _need(vcache, "vcache", kcache.shape, q.dtype)
    _need(kbar, "kbar", dtype=q.dtype)
    slots = n_init + n_local + topk
    _need(idx_in, "idx_in", (B, Hkv, slots), torch.int32)
    _need(idx_out, "idx_out", (B, Hkv, slots), torch.int32)
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype)
    need = sparse_decode_workspace_bytes(B, H, Hkv, pos, topk, n_init, n_local, d, block)
    if workspace is None:  # zero-filled: its first words are counters that must start at zero
        workspace = torch.zeros(max(need, 256), device=q.device, dtype=torch.uint8)
    fn = _lib.sala_sparse_decode_pdl if pdl else _lib.sala_sparse_decode
    _check(fn(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(kbar), _ptr(idx_in), _ptr(idx_out),
              _ptr(o), B, H, Hkv, pos, Tmax, kbar.shape[2], d, block, topk, n_init, n_local,
              float(scale), _ptr(workspace), workspace.numel(), _dt(q), _stream(stream)),
           "sala_sparse_decode_pdl" if pdl else "sala_sparse_decode")
    return o


def sparse_decode_paged_workspace_bytes(B, H, Hkv, max_pos, topk, n_init, n_local, d, block=64):
    return _lib.sala_sparse_decode_paged_workspace(B, H, Hkv, max_pos, block, topk, n_init, n_local, d)


def sparse_decode_paged(q, k_pages, v_pages, page_table, kbar, pos, max_pos, topk, n_init, n_local,
                        idx_out=None, o=None, scale=0.0, workspace=None, stream=None):
    """One query token per head for each of B sequences at its own position pos[b] (an int32
    device tensor, each <= max_pos), the KV cache in pages: k_pages, v_pages [n_pages, Hkv, 64, d],
    page_table [B, max_pages] int32.  q: [B, H, d]; kbar [B, Hkv, nb_cap, d].  Returns o."""
    B, H, d = q.shape
    n_pages, Hkv = k_pages.shape[0], k_pages.shape[1]
    _need(q, "q"); _need(k_pages, "k_pages", dtype=q.dtype)
    _need(v_pages, "v_pages", k_pages.shape, q.dtype)
    assert k_pages.shape[2:] == (64, d), k_pages.shape
    _need(page_table, "page_table", dtype=torch.int32)
    assert page_table.dim() == 2 and page_table.shape[0] == B
    _need(pos, "pos", (B,), torch.int32)
    _need(kbar, "kbar", dtype=q.dtype)
    slots = n_init + n_local + topk
    _need(idx_out, "idx_out", (B, Hkv, slots), torch.int32)
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", q.shape, q.dtype)
    need = sparse_decode_paged_workspace_bytes(B, H, Hkv, max_pos, topk, n_init, n_local, d)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(_lib.sala_sparse_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), n_pages,
                                         _ptr(page_table), page_table.shape[1], _ptr(kbar),
                                         kbar.shape[2], _ptr(pos), int(max_pos), _ptr(idx_out),
                                         _ptr(o), B, H, Hkv, d, 64, topk, n_init, n_local,
                                         ctypes.c_float(scale), _ptr(workspace), workspace.numel(),
                                         _dt(q), _stream(stream)), "sala_sparse_decode_paged")
    return o


def debug_bounds_build() -> bool:
    """Whether the loaded library is the bounds-checking build."""
    return bool(_lib.sala_debug_bounds_build())


def check_status(stream=None):
    """Synchronise the stream and raise if a kernel recorded a device-side fault."""
    _check(_lib.sala_check_status(_stream(stream)), "sala_check_status")


def set_wait_limit_ns(ns: int):
    _lib.sala_set_wait_limit_ns(int(ns))


def selftest_wait_timeout(stream=None):
    _check(_lib.sala_selftest_wait_timeout(_stream(stream)), "sala_selftest_wait_timeout")


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


raw = _lib  # the loaded C library, for callers that marshal pointers themselves
