"""fp64 CPU oracle for the SALA hybrid attention forward.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` are the only callers.  The product path (``hybrid_sparse_linear_b200``) never imports
this package, and this package never imports the product.

The arithmetic lives in ``sala_oracle.cpp`` (plain loops, fp64); this module only marshals numpy
arrays through ctypes.  Every function takes float64 arrays in the row-major layouts documented in
the C source: ``q, k, v`` are ``[B, heads, rows, dim]``.  ``from_tensor`` turns a torch tensor of
any dtype the GPU path uses (bf16, fp32) into the exact float64 values it holds.

Pinned by ``tests/test_oracle_*.py`` (closed forms, brute force, invariants between independent
forms); see the module docstrings there for which pin covers which function.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sala_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liborc.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)
_i = ctypes.c_int
_l = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (fp64, -O2, no fast-math) into ``oracle/liborc.so``."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.orc_round_bf16.restype = ctypes.c_double
            lib.orc_round_bf16.argtypes = [ctypes.c_double]
            lib.orc_linear_recurrent.argtypes = [_D, _D, _D, _D, _D, _D, _D, _i, _i, _i, _i, _i, _i]
            lib.orc_linear_quadratic.argtypes = [_D, _D, _D, _D, _D, _D, _i, _i, _i, _i, _i, _I64, _l, _i]
            lib.orc_linear_chunked.argtypes = [_D, _D, _D, _D, _D, _D, _D, _i, _i, _i, _i, _i, _i, _i]
            lib.orc_linear_decode.argtypes = [_D, _D, _D, _D, _D, _D, _i, _i, _i, _i]
            lib.orc_rope.argtypes = [_D, _i, _i, _i, _i, _l, ctypes.c_double]
            lib.orc_qk_norm.argtypes = [_D, _l, _i, ctypes.c_double]
            lib.orc_block_compress.argtypes = [_D, _D, _i, _i, _i, _i, _i, _i, _i, _i]
            lib.orc_block_scores_at.argtypes = [_D, _D, _I64, _l, _D, _i, _i, _i, _i, _i]
            lib.orc_block_select.argtypes = [_D, _D, _I32, _D, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                             _i, _i, _i, _i]
            lib.orc_block_select_qblock.argtypes = [_D, _D, _I32, _D] + [_i] * 12
            lib.orc_block_select_qblock_softmax.argtypes = [_D, _D, _I32, _D] + [_i] * 11 + [
                ctypes.c_double, _i]
            lib.orc_sparse_attention.argtypes = [_D, _D, _D, _I32, _D, _i, _i, _i, _i, _i, _i, _i,
                                                 _i, _i, ctypes.c_double, _I64, _l, _i]
            lib.orc_dense_causal_attention.argtypes = [_D, _D, _D, _D, _i, _i, _i, _i, _i, _i, _i,
                                                       ctypes.c_double, _i]
            for name in ("orc_linear_recurrent", "orc_linear_quadratic", "orc_linear_chunked",
                         "orc_linear_decode", "orc_qk_norm", "orc_block_compress", "orc_block_scores_at",
                         "orc_block_select", "orc_sparse_attention", "orc_dense_causal_attention"):
                getattr(lib, name).restype = None
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def from_tensor(t) -> np.ndarray:
    """Exact float64 copy of a torch tensor (bf16 and fp32 values are exact in fp64)."""
    import torch
    return t.detach().to("cpu", torch.float64).contiguous().numpy()


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(_D)


def round_bf16(x):
    """bf16 round-to-nearest-even of float64 values (elementwise)."""
    lib = _load()
    x = np.asarray(x, dtype=np.float64)
    return np.vectorize(lib.orc_round_bf16, otypes=[np.float64])(x) if x.ndim else \
        lib.orc_round_bf16(float(x))


# ----------------------------------------------------------------------------------------------
# Linear attention

def _lin_args(q, k, v, lam, s_in):
    q, k, v, lam = _f64(q), _f64(k), _f64(v), _f64(lam)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, N, dk) and v.shape == (B, H, N, dv) and lam.shape == (H,)
    s_in = None if s_in is None else _f64(s_in)
    if s_in is not None:
        assert s_in.shape == (B, H, dk, dv)
    return q, k, v, lam, s_in, B, H, N, dk, dv


def linear_recurrent(q, k, v, lam, s_in=None, threads=None):
    """Recurrent form: S <- lambda S + k^T v; o = q S.  Returns (o, s_out)."""
    q, k, v, lam, s_in, B, H, N, dk, dv = _lin_args(q, k, v, lam, s_in)
    o = np.empty((B, H, N, dv)); s_out = np.empty((B, H, dk, dv))
    _load().orc_linear_recurrent(_p(q), _p(k), _p(v), _p(lam), _p(s_in), _p(o), _p(s_out),
                                 B, H, N, dk, dv, threads or default_threads())
    return o, s_out


def linear_quadratic(q, k, v, lam, s_in=None, rows=None, threads=None):
    """Quadratic form.  rows: optional int array [n, 2] of (b*H + h, token); returns [n, dv]."""
    q, k, v, lam, s_in, B, H, N, dk, dv = _lin_args(q, k, v, lam, s_in)
    if rows is None:
        o = np.empty((B, H, N, dv)); rp = None; n = 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
        n = rows.shape[0]; o = np.empty((n, dv)); rp = rows.ctypes.data_as(_I64)
    _load().orc_linear_quadratic(_p(q), _p(k), _p(v), _p(lam), _p(s_in), _p(o), B, H, N, dk, dv,
                                 rp, n, threads or default_threads())
    return o


def linear_chunked(q, k, v, lam, chunk, s_in=None, threads=None):
    """Chunked form (intra-chunk mask + carried state).  Returns (o, s_out)."""
    q, k, v, lam, s_in, B, H, N, dk, dv = _lin_args(q, k, v, lam, s_in)
    o = np.empty((B, H, N, dv)); s_out = np.empty((B, H, dk, dv))
    _load().orc_linear_chunked(_p(q), _p(k), _p(v), _p(lam), _p(s_in), _p(o), _p(s_out),
                               B, H, N, dk, dv, int(chunk), threads or default_threads())
    return o, s_out


def linear_backward(q, k, v, lam, do):
    """Gradients (dq, dk, dv) of sum(o * do), o the linear attention of a fresh sequence (no
    carried state), by fp64 autograd through the plain quadratic form
    o = ((Q K^T) * Dmask) V with Dmask[i, j] = lam^(i - j) for j <= i, 0 above the diagonal.
    (plain PyTorch CPU ops; the contract's backward pass of the linear layers.)"""
    import torch
    t = lambda x: torch.tensor(_f64(x), dtype=torch.float64)
    Q, K, V, dO = (t(x).requires_grad_(r) for x, r in ((q, True), (k, True), (v, True), (do, False)))
    lam_t = t(lam)
    N = Q.shape[2]
    i = torch.arange(N, dtype=torch.float64)
    diff = i[:, None] - i[None, :]
    causal = diff >= 0
    Dm = torch.where(causal, lam_t[:, None, None] ** diff.clamp(min=0), torch.zeros(()))  # [H, N, N]
    A = (Q @ K.transpose(-1, -2)) * Dm
    O = A @ V
    (O * dO).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def linear_decode(q, k, v, lam, state):
    """One decode step.  q,k: [B,H,dk]; v: [B,H,dv]; state [B,H,dk,dv].  Returns (o, new_state)."""
    q, k, v, lam = _f64(q), _f64(k), _f64(v), _f64(lam)
    S = _f64(state).copy()
    B, H, dk, dv = S.shape
    o = np.empty((B, H, dv))
    _load().orc_linear_decode(_p(q), _p(k), _p(v), _p(lam), _p(S), _p(o), B, H, dk, dv)
    return o, S


def rope(x, pos0=0, base=10000.0):
    """Rotary position embedding of x [B,H,N,d] (row r at position pos0 + r); a rotated copy.
    The linear layers apply it to q and k before the linear attention (HyPE)."""
    x = _f64(x).copy()
    B, H, N, d = x.shape
    assert d % 2 == 0
    _load().orc_rope(_p(x), B, H, N, d, int(pos0), float(base))
    return x


def qk_norm(x, eps=1e-6):
    """Weight-free RMS normalisation of every head row of x [..., d] (QK normalisation); a
    normalised copy."""
    x = _f64(x).copy()
    d = x.shape[-1]
    _load().orc_qk_norm(_p(x), int(x.size // d), d, float(eps))
    return x


def linear_chunked_rope(q, k, v, lam, chunk, pos0=0, base=10000.0, s_in=None):
    """Linear attention of a linear (HyPE) layer: q and k rotated by position first.  Returns
    (o, s_out) as linear_chunked."""
    return linear_chunked(rope(q, pos0, base), rope(k, pos0, base), v, lam, chunk, s_in=s_in)


# ----------------------------------------------------------------------------------------------
# Sparse attention

def block_compress(k, block, first_block=0, n_blocks=None, round_to_bf16=True):
    """Mean of each complete block of keys, rounded once to bf16.  k: [B,Hkv,N,d]."""
    k = _f64(k)
    B, Hkv, N, d = k.shape
    if n_blocks is None:
        n_blocks = N // block - first_block
    assert 0 <= first_block and (first_block + n_blocks) * block <= N
    out = np.empty((B, Hkv, n_blocks, d))
    _load().orc_block_compress(_p(k), _p(out), B, Hkv, N, d, block, first_block, n_blocks,
                               1 if round_to_bf16 else 0)
    return out


def block_select(q, kbar, block, topk, n_init, n_local, q_pos0=0, slots=None, threads=None):
    """Per (batch, KV group, query row) block selection.  Returns (idx int32, kth_score)."""
    q, kbar = _f64(q), _f64(kbar)
    B, H, Nq, d = q.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    slots = slots or (n_init + n_local + topk)
    idx = np.empty((B, Hkv, Nq, slots), dtype=np.int32)
    kth = np.empty((B, Hkv, Nq))
    _load().orc_block_select(_p(q), _p(kbar), idx.ctypes.data_as(_I32), _p(kth), B, H, Hkv, Nq,
                             int(q_pos0), nb, d, block, topk, n_init, n_local, slots,
                             threads or default_threads())
    return idx, kth


def block_select_qblock(q, kbar, block, topk, n_init, n_local, slots=None, threads=None):
    """One selection per (batch, KV group, query block of `block` tokens), written to every token
    row of the block.  Returns (idx int32 [B,Hkv,Nq,slots], kth_score [B,Hkv,Nq])."""
    q, kbar = _f64(q), _f64(kbar)
    B, H, Nq, d = q.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    slots = slots or (n_init + n_local + topk)
    idx = np.empty((B, Hkv, Nq, slots), dtype=np.int32)
    kth = np.empty((B, Hkv, Nq))
    _load().orc_block_select_qblock(_p(q), _p(kbar), idx.ctypes.data_as(_I32), _p(kth), B, H, Hkv,
                                    Nq, nb, d, block, topk, n_init, n_local, slots,
                                    threads or default_threads())
    return idx, kth


def block_select_qblock_softmax(q, kbar, block, topk, n_init, n_local, slots=None, scale=None,
                                threads=None):
    """Query-block selection scored by softmax-probability group aggregation: per head, the
    block's mean query gives logits scale * (u_h . kbar_j) over the candidates, a softmax over
    them, the probabilities summed over the group's heads.  Returns (idx, kth_score) as
    block_select_qblock; scale defaults to 1/sqrt(d)."""
    q, kbar = _f64(q), _f64(kbar)
    B, H, Nq, d = q.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    slots = slots or (n_init + n_local + topk)
    scale = (1.0 / np.sqrt(d)) if scale is None else float(scale)
    idx = np.empty((B, Hkv, Nq, slots), dtype=np.int32)
    kth = np.empty((B, Hkv, Nq))
    _load().orc_block_select_qblock_softmax(_p(q), _p(kbar), idx.ctypes.data_as(_I32), _p(kth), B,
                                            H, Hkv, Nq, nb, d, block, topk, n_init, n_local, slots,
                                            scale, threads or default_threads())
    return idx, kth


def qblock_sum(q, block):
    """q with every token replaced by the per-head sum of q over its query block (plain numpy):
    the query tensor whose per-token selection is the query-block selection."""
    q = _f64(q)
    B, H, Nq, d = q.shape
    out = np.empty_like(q)
    for r0 in range(0, Nq, block):
        out[:, :, r0:r0 + block] = q[:, :, r0:r0 + block].sum(axis=2, keepdims=True)
    return out


def block_scores_at(q, kbar, quads):
    """Scores for (b, g, r, block) quadruples (int array [n, 4])."""
    q, kbar = _f64(q), _f64(kbar)
    B, H, Nq, d = q.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    quads = np.ascontiguousarray(quads, dtype=np.int64).reshape(-1, 4)
    out = np.empty(quads.shape[0])
    _load().orc_block_scores_at(_p(q), _p(kbar), quads.ctypes.data_as(_I64), quads.shape[0],
                                _p(out), H, Hkv, Nq, nb, d)
    return out


def sparse_attention(q, k, v, idx, block, scale=None, q_pos0=0, rows=None, threads=None):
    """Softmax attention over the selected blocks.  rows: optional [n, 2] of (b*H + h, r)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    slots = idx.shape[-1]
    scale = (1.0 / np.sqrt(d)) if scale is None else float(scale)
    if rows is None:
        o = np.empty((B, H, Nq, d)); rp = None; n = 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
        n = rows.shape[0]; o = np.empty((n, d)); rp = rows.ctypes.data_as(_I64)
    _load().orc_sparse_attention(_p(q), _p(k), _p(v), idx.ctypes.data_as(_I32), _p(o), B, H, Hkv,
                                 Nq, int(q_pos0), Nk, d, block, slots, scale, rp, n,
                                 threads or default_threads())
    return o


def block_select_per_head(q, kbar, block, topk, n_init, n_local, q_pos0=0, slots=None, threads=None):
    """Per-query-head block selection (a listed variant of the selection step): every query head h
    chooses its own blocks, scored with its own query, score_h(j) = q_h . kbar_{g(h), j}; forced
    blocks, candidates, ties and the row layout as block_select.  This is block_select with groups of
    one head: each head gets its KV head's kbar.  Returns (idx [B, H, Nq, slots] int32, kth_score
    [B, H, Nq])."""
    q, kbar = _f64(q), _f64(kbar)
    B, H, Nq, d = q.shape
    Hkv = kbar.shape[1]
    G = H // Hkv
    kbar_h = np.ascontiguousarray(np.repeat(kbar, G, axis=1))   # [B, H, nb, d]: head h -> kbar of h // G
    return block_select(q, kbar_h, block, topk, n_init, n_local, q_pos0=q_pos0, slots=slots,
                        threads=threads)


def sparse_attention_per_head(q, k, v, idx_h, block, scale=None, q_pos0=0, threads=None):
    """Softmax attention over per-head selections: idx_h [B, H, Nq, slots] gives query head h its
    own blocks (of its KV head's keys).  One sparse_attention per head, each a group of one head."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    idx_h = np.ascontiguousarray(idx_h, dtype=np.int32)
    o = np.empty((B, H, Nq, d))
    for h in range(H):
        g = h // G
        o[:, h:h + 1] = sparse_attention(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1],
                                         idx_h[:, h:h + 1], block, scale=scale, q_pos0=q_pos0,
                                         threads=threads)
    return o


def dense_causal_attention(q, k, v, scale=None, q_pos0=0, threads=None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    scale = (1.0 / np.sqrt(d)) if scale is None else float(scale)
    o = np.empty((B, H, Nq, d))
    _load().orc_dense_causal_attention(_p(q), _p(k), _p(v), _p(o), B, H, Hkv, Nq, int(q_pos0), Nk,
                                       d, scale, threads or default_threads())
    return o


def _visible(idx_bg, N, block):
    """[N, N] bool: key j visible to query row i (prefill, rows at positions 0..N-1) iff j's block
    is in row i's selection and j <= i."""
    import torch
    nb = (N + block - 1) // block
    sel = torch.zeros((N, nb + 1), dtype=torch.bool)
    ids = torch.as_tensor(np.asarray(idx_bg, dtype=np.int64))
    ids = torch.where(ids >= 0, ids, torch.full_like(ids, nb))  # padding -> a dummy column
    sel.scatter_(1, ids, True)
    j = torch.arange(N)
    return sel[:, j // block] & (j[None, :] <= j[:, None])


def sparse_lse(q, k, idx, block, scale=None):
    """Natural log-sum-exp of each prefill row's visible logits scale * (q_i . k_j): [B, H, N]
    (-inf where a row sees no key).  Plain PyTorch fp64."""
    import torch
    q, k = _f64(q), _f64(k)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    scale = (1.0 / np.sqrt(d)) if scale is None else float(scale)
    out = np.empty((B, H, N))
    for b in range(B):
        for g in range(Hkv):
            vis = _visible(idx[b, g], N, block)
            K = torch.from_numpy(k[b, g])
            for h in range(g * G, (g + 1) * G):
                s = scale * (torch.from_numpy(q[b, h]) @ K.T)
                out[b, h] = torch.logsumexp(s.masked_fill(~vis, -np.inf), dim=1).numpy()
    return out


def sparse_attention_backward(q, k, v, idx, do, block, scale=None):
    """Gradients (dq, dk, dv) of sum(o * do), o the sparse attention of a prefill (rows at
    positions 0..N-1) over the selected blocks idx [B, Hkv, N, slots], the selection held fixed
    (the top-k choice is piecewise constant in q and k and passes no gradient).  fp64 autograd
    through the plain masked softmax o_i = softmax_j(scale q_i . k_j, j visible) V, one query
    head at a time; dk and dv sum the G heads of a KV group.  Every row must see a key.
    (plain PyTorch CPU ops; the backward pass of the sparse layers.)"""
    import torch
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    scale = (1.0 / np.sqrt(d)) if scale is None else float(scale)
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for g in range(Hkv):
            vis = _visible(idx[b, g], N, block)
            assert bool(vis.any(dim=1).all()), "a query row sees no key"
            for h in range(g * G, (g + 1) * G):
                Q = torch.tensor(q[b, h], requires_grad=True)
                K = torch.tensor(k[b, g], requires_grad=True)
                V = torch.tensor(v[b, g], requires_grad=True)
                s = (scale * (Q @ K.T)).masked_fill(~vis, -np.inf)
                o = torch.softmax(s, dim=1) @ V
                gq, gk, gv = torch.autograd.grad((o * torch.from_numpy(do[b, h])).sum(), (Q, K, V))
                dq[b, h] = gq.numpy()
                dk[b, g] += gk.numpy()
                dv[b, g] += gv.numpy()
    return dq, dk, dv


def sparse_dq_rows(q, k, v, idx, do, block, rows, scale=None):
    """dq of selected prefill rows only, rows: [n, 3] of (b, h, i): for each, fp64 autograd of
    o_i . do_i through the softmax over row i's visible keys (its selected blocks, keys <= i).
    Equals the rows of sparse_attention_backward's dq; cheap at any N."""
    import torch
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    scale = (1.0 / np.sqrt(d)) if scale is None else float(scale)
    out = np.empty((len(rows), d))
    for n, (b, h, i) in enumerate(np.asarray(rows, dtype=np.int64)):
        g = h // G
        blks = [int(x) for x in np.asarray(idx[b, g, i]) if x >= 0]
        keys = np.concatenate([np.arange(x * block, min((x + 1) * block, i + 1)) for x in blks])
        Q = torch.tensor(_f64(q[b, h, i]), requires_grad=True)
        K = torch.from_numpy(_f64(k[b, g, keys]))
        V = torch.from_numpy(_f64(v[b, g, keys]))
        o = torch.softmax(scale * (K @ Q), dim=0) @ V
        (gq,) = torch.autograd.grad((o * torch.from_numpy(_f64(do[b, h, i]))).sum(), (Q,))
        out[n] = gq.numpy()
    return out


def qblock_softmax_scores(q, kbar, block, b, g, c, n_init, n_local, scale=None):
    """Scores of block_select_qblock_softmax's candidates n_init .. c - n_local for one (batch,
    KV group, query block), plain numpy fp64: (candidate block ids, scores)."""
    q, kbar = _f64(q), _f64(kbar)
    B, H, Nq, d = q.shape
    Hkv = kbar.shape[1]
    G = H // Hkv
    scale = (1.0 / np.sqrt(d)) if scale is None else float(scale)
    u = q[b, g * G:(g + 1) * G, c * block:min(Nq, (c + 1) * block)].mean(axis=1)   # [G, d]
    ids = np.arange(n_init, c - n_local + 1)
    logits = scale * u @ kbar[b, g, ids].T                                          # [G, nc]
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    return ids, (p / p.sum(axis=1, keepdims=True)).sum(axis=0)
