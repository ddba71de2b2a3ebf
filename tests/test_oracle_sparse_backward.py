"""Pins of the oracle's backward pass of the sparse attention (gradients of sum(o * do) with the
selection held fixed) and of its per-row log-sum-exp.  CPU only.

* central finite differences of the pinned C forward (oracle.sparse_attention) at every element
  of q, k and v, on a case whose selection masks different blocks for different rows;
* full selection (k >= every candidate): equals torch's scaled_dot_product_attention (causal) in
  fp64 autograd, with the group's heads sharing K and V;
* identities of softmax attention: per KV group, sum_j dk_j = 0 (each row's dS sums to zero) and
  sum_j dv_j = sum over the group's heads and rows of do (each row's P sums to one); keys that are
  all equal give dq = 0.  A dropped D_i term, a transposed P or a wrong head-to-group map fails;
* lse: o_i = sum_j exp(scale q_i.k_j - lse_i) v_j over the visible keys reproduces the C forward,
  and row 0 (one visible key) has lse = scale q_0.k_0.
"""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _case(B, H, Hkv, N, d, block, topk, seed, n_init=1, n_local=1):
    q, k, v, do = (_rand(s, seed + i) for i, s in
                   enumerate([(B, H, N, d), (B, Hkv, N, d), (B, Hkv, N, d), (B, H, N, d)]))
    kbar = oracle.block_compress(k, block, round_to_bf16=False)
    idx = oracle.block_select(q, kbar, block, topk, n_init, n_local)[0]
    return q, k, v, do, idx


def test_finite_differences():
    B, H, Hkv, N, d, block = 1, 2, 1, 40, 4, 8
    q, k, v, do, idx = _case(B, H, Hkv, N, d, block, 1, 11)
    # the selection must actually leave blocks out for some rows
    assert (idx[0, 0, 30:] >= 0).sum(axis=1).max() < 30 // block + 1
    dq, dk, dv = oracle.sparse_attention_backward(q, k, v, idx, do, block)
    f = lambda q_, k_, v_: float(np.sum(oracle.sparse_attention(q_, k_, v_, idx, block, threads=1) * do))
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for ix in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[ix] += h
            xm[ix] -= h
            ap = [xp if name == n else y for n, y in (("q", q), ("k", k), ("v", v))]
            am = [xm if name == n else y for n, y in (("q", q), ("k", k), ("v", v))]
            num[ix] = (f(*ap) - f(*am)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_full_selection_matches_sdpa():
    B, H, Hkv, N, d, block = 2, 4, 2, 48, 8, 8
    q, k, v, do, idx = _case(B, H, Hkv, N, d, block, N // block, 21)
    dq, dk, dv = oracle.sparse_attention_backward(q, k, v, idx, do, block)
    G = H // Hkv
    Q = torch.tensor(q, requires_grad=True)
    K = torch.tensor(k, requires_grad=True)
    V = torch.tensor(v, requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(
        Q, K.repeat_interleave(G, dim=1), V.repeat_interleave(G, dim=1), is_causal=True)
    gq, gk, gv = torch.autograd.grad((o * torch.from_numpy(do)).sum(), (Q, K, V))
    np.testing.assert_allclose(dq, gq.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, gk.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, gv.numpy(), rtol=1e-10, atol=1e-12)


def test_softmax_identities():
    B, H, Hkv, N, d, block = 1, 6, 2, 72, 8, 8
    q, k, v, do, idx = _case(B, H, Hkv, N, d, block, 2, 31)
    dq, dk, dv = oracle.sparse_attention_backward(q, k, v, idx, do, block)
    G = H // Hkv
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
    for g in range(Hkv):
        np.testing.assert_allclose(dv[:, g].sum(axis=1), do[:, g * G:(g + 1) * G].sum(axis=(1, 2)),
                                   rtol=1e-12, atol=1e-11)
    # equal keys: every visible logit of a row is the same, so the logits' gradient is zero
    ke = np.broadcast_to(_rand((B, Hkv, 1, d), 32), k.shape).copy()
    dq_e, _, _ = oracle.sparse_attention_backward(q, ke, v, idx, do, block)
    np.testing.assert_allclose(dq_e, 0.0, atol=1e-12)


def test_lse_reproduces_forward():
    B, H, Hkv, N, d, block = 1, 4, 2, 56, 8, 8
    q, k, v, _, idx = _case(B, H, Hkv, N, d, block, 2, 41)
    scale = 1.0 / np.sqrt(d)
    lse = oracle.sparse_lse(q, k, idx, block)
    o_ref = oracle.sparse_attention(q, k, v, idx, block)
    G = H // Hkv
    for b in range(B):
        for h in range(H):
            g = h // G
            vis = oracle._visible(idx[b, g], N, block).numpy()
            p = np.where(vis, np.exp(scale * q[b, h] @ k[b, g].T - lse[b, h][:, None]), 0.0)
            np.testing.assert_allclose(p @ v[b, g], o_ref[b, h], rtol=1e-12, atol=1e-12)
            assert lse[b, h, 0] == pytest.approx(scale * q[b, h, 0] @ k[b, g, 0], rel=1e-14)


def test_sampled_dq_rows_equal_full_backward():
    B, H, Hkv, N, d, block = 2, 4, 2, 80, 8, 16
    q, k, v, do, idx = _case(B, H, Hkv, N, d, block, 2, 51)
    dq = oracle.sparse_attention_backward(q, k, v, idx, do, block)[0]
    rows = np.array([[0, 0, 0], [1, 3, 79], [0, 2, 40], [1, 1, 17], [0, 3, 63], [1, 0, 64]])
    got = oracle.sparse_dq_rows(q, k, v, idx, do, block, rows)
    np.testing.assert_allclose(got, dq[rows[:, 0], rows[:, 1], rows[:, 2]], rtol=1e-12, atol=1e-13)
