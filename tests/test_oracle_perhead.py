"""Pins for the oracle's per-query-head block selection and the attention over it.

* brute force: every (batch, head, row) of a small random case against a plain sort of the head's
  own scores q_h . kbar_g(h) over the candidates (ties to the lower block), plus the forced blocks;
* heads of a group that carry the same query choose exactly the group's selection (summing G equal
  queries multiplies every score by G > 0, which keeps the order);
* a hand case where two heads of one group want different blocks and the group sum picks a third;
* attention: per-head selections that agree within each group give the group attention; a head's
  output depends only on its own selection.
"""
import numpy as np

import oracle


def _brute(q, kbar, T, topk, n_init, n_local, q_pos0=0):
    B, H, Nq, d = q.shape
    Hkv = kbar.shape[1]
    G = H // Hkv
    slots = n_init + n_local + topk
    out = np.full((B, H, Nq, slots), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for r in range(Nq):
                c = (q_pos0 + r) // T
                forced = set(range(min(n_init, c + 1))) | set(range(max(0, c - n_local + 1), c + 1))
                cand = [j for j in range(n_init, c - n_local + 1)]
                sc = [(-(q[b, h, r] @ kbar[b, h // G, j]), j) for j in cand]
                sc.sort()
                sel = sorted(forced | {j for _, j in sc[:topk]})
                out[b, h, r, :len(sel)] = sel
    return out


def test_per_head_selection_brute_force():
    rng = np.random.default_rng(41)
    B, H, Hkv, T, d, N = 2, 6, 2, 4, 5, 13 * 4 + 3
    q = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    kbar = oracle.block_compress(k, T)
    for topk, n_init, n_local in [(3, 1, 1), (2, 1, 2), (5, 0, 1)]:
        idx, kth = oracle.block_select_per_head(q, kbar, T, topk, n_init, n_local)
        np.testing.assert_array_equal(idx, _brute(q, kbar, T, topk, n_init, n_local))
        assert kth.shape == (B, H, N)


def test_equal_heads_choose_the_group_selection():
    rng = np.random.default_rng(42)
    B, Hkv, G, T, d, N = 1, 2, 4, 4, 6, 60
    base = rng.standard_normal((B, Hkv, 1, N, d))
    q = np.repeat(base, G, axis=2).reshape(B, Hkv * G, N, d)
    kbar = oracle.block_compress(rng.standard_normal((B, Hkv, N, d)), T)
    ih, _ = oracle.block_select_per_head(q, kbar, T, 3, 1, 2)
    ig, _ = oracle.block_select(q, kbar, T, 3, 1, 2)
    for h in range(Hkv * G):
        np.testing.assert_array_equal(ih[:, h], ig[:, h // G])


def test_hand_case_heads_disagree_with_their_sum():
    # one group of two heads, d = 2, block 1, query at position 4 (block 4), n_local 1, top-1:
    # candidates 1, 2, 3 with kbar (1, 0), (0, 1), (0.8, 0.8);
    # head 0 = (1, 0) picks block 1 (score 1 > 0.8 > 0), head 1 = (0, 1) picks block 2,
    # the group sum (1, 1) scores 1, 1, 1.6 and picks block 3.
    kbar = np.zeros((1, 1, 5, 2))
    kbar[0, 0, 1] = (1.0, 0.0)
    kbar[0, 0, 2] = (0.0, 1.0)
    kbar[0, 0, 3] = (0.8, 0.8)
    q = np.zeros((1, 2, 1, 2))
    q[0, 0, 0] = (1.0, 0.0)
    q[0, 1, 0] = (0.0, 1.0)
    ih, kth = oracle.block_select_per_head(q, kbar, 1, 1, 1, 1, q_pos0=4)
    assert list(ih[0, 0, 0]) == [0, 1, 4]
    assert list(ih[0, 1, 0]) == [0, 2, 4]
    assert kth[0, 0, 0] == 1.0 and kth[0, 1, 0] == 1.0
    ig, _ = oracle.block_select(q, kbar, 1, 1, 1, 1, q_pos0=4)
    assert list(ig[0, 0, 0]) == [0, 3, 4]


def test_per_head_attention_reduces_to_group_attention():
    rng = np.random.default_rng(43)
    B, H, Hkv, T, d, N = 1, 4, 2, 4, 8, 40
    q = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    kbar = oracle.block_compress(k, T)
    ig, _ = oracle.block_select(q, kbar, T, 2, 1, 1)
    G = H // Hkv
    ih = np.repeat(ig, G, axis=1)
    np.testing.assert_allclose(oracle.sparse_attention_per_head(q, k, v, ih, T),
                               oracle.sparse_attention(q, k, v, ig, T), rtol=0, atol=1e-14)
    # changing one head's selection changes only that head's output
    ih2 = ih.copy()
    ih2[:, 1, 20:] = np.where(ih2[:, 1, 20:] == 1, 0, ih2[:, 1, 20:])
    o1 = oracle.sparse_attention_per_head(q, k, v, ih, T)
    o2 = oracle.sparse_attention_per_head(q, k, v, ih2, T)
    np.testing.assert_array_equal(np.delete(o1, 1, axis=1), np.delete(o2, 1, axis=1))
