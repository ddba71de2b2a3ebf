"""Pins of the oracle's query-block selection with softmax-probability group aggregation.  CPU only.

* a hand-worked case where the aggregation and the summed-query score disagree: one head certain
  about block 0, two heads fairly sure of block 1 -- probabilities summed pick block 1, logits
  summed pick block 0 (so the heads are not merged before the softmax);
* one head per group: a softmax is monotone in its logits, so the choice equals the plain
  query-block selection (summed query) on the same inputs;
* invariances: adding one vector to every k-bar shifts each head's logits by a constant (the
  softmax ignores it); permuting the heads of a group changes nothing;
* scale 0: every head's probabilities are exactly uniform, all scores tie, and the lowest
  candidates win (the tie rule).
"""
import numpy as np

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_hand_case_heads_disagree():
    # block size 1: query block c is token c; token 3's candidates are blocks 0, 1, 2
    d, N = 3, 4
    q = np.zeros((1, 3, N, d))
    q[0, 0, 3] = [20.0, 0.0, 0.0]
    q[0, 1, 3] = [0.0, 2.0, -5.0]
    q[0, 2, 3] = [0.0, 2.0, -5.0]
    kbar = np.zeros((1, 1, N, d))
    kbar[0, 0, 0] = [1.0, 0.0, 0.0]
    kbar[0, 0, 1] = [0.0, 1.0, 0.0]
    kbar[0, 0, 2] = [0.0, 0.0, 1.0]
    idx, kth = oracle.block_select_qblock_softmax(q, kbar, 1, 1, 0, 1, scale=1.0)
    assert list(idx[0, 0, 3]) == [1, 3]
    # block 1's score: 2 * e^2 / (1 + e^2 + e^-5) + e^0 / (e^20 + 2)
    p1 = 2 * np.exp(2) / (1 + np.exp(2) + np.exp(-5)) + 1 / (np.exp(20) + 2)
    assert abs(kth[0, 0, 3] - p1) < 1e-12
    idx_sum, _ = oracle.block_select_qblock(q, kbar, 1, 1, 0, 1)
    assert list(idx_sum[0, 0, 3]) == [0, 3]


def test_one_head_per_group_equals_summed_query_selection():
    q = _rand((2, 3, 700, 16), 1)
    kbar = _rand((2, 3, 11, 16), 2)
    for topk in (1, 3, 20):
        a, _ = oracle.block_select_qblock_softmax(q, kbar, 64, topk, 1, 2)
        b, _ = oracle.block_select_qblock(q, kbar, 64, topk, 1, 2)
        np.testing.assert_array_equal(a, b)


def test_invariances():
    q = _rand((1, 8, 900, 16), 3)
    kbar = _rand((1, 2, 15, 16), 4)
    a, _ = oracle.block_select_qblock_softmax(q, kbar, 64, 3, 1, 2)
    shifted = kbar + _rand((1, 1, 1, 16), 5)
    b, _ = oracle.block_select_qblock_softmax(q, shifted, 64, 3, 1, 2)
    np.testing.assert_array_equal(a, b)
    perm = np.concatenate([np.random.default_rng(6).permutation(4), 4 + np.random.default_rng(7).permutation(4)])
    c, _ = oracle.block_select_qblock_softmax(q[:, perm], kbar, 64, 3, 1, 2)
    np.testing.assert_array_equal(a, c)


def test_zero_scale_ties_to_lowest_blocks():
    q = _rand((1, 4, 64 * 12, 8), 8)
    kbar = _rand((1, 2, 12, 8), 9)
    idx, kth = oracle.block_select_qblock_softmax(q, kbar, 64, 3, 1, 2, scale=0.0)
    # block c = 11: candidates 1 .. 9, all scoring G / 9; the lowest three win
    assert list(idx[0, 0, 64 * 11]) == [0, 1, 2, 3, 10, 11]
    assert abs(kth[0, 0, 64 * 11] - 2 / 9) < 1e-12


def test_numpy_scores_agree_with_the_selection():
    q = _rand((2, 6, 64 * 20 + 9, 16), 10)
    kbar = _rand((2, 2, 21, 16), 11)
    topk, n_init, n_local = 4, 1, 2
    idx, kth = oracle.block_select_qblock_softmax(q, kbar, 64, topk, n_init, n_local)
    for b in range(2):
        for g in range(2):
            for c in (3, 9, 20):
                ids, sc = oracle.qblock_softmax_scores(q, kbar, 64, b, g, c, n_init, n_local)
                assert abs(sc.sum() - 3.0) < 1e-12  # G heads, each a distribution
                best = ids[np.lexsort((ids, -sc))][:topk]
                forced = {0} | set(range(c - n_local + 1, c + 1))
                assert sorted(forced | set(best.tolist())) == [x for x in idx[b, g, 64 * c] if x >= 0]
                if len(ids) >= topk:
                    assert abs(np.sort(sc)[::-1][topk - 1] - kth[b, g, 64 * c]) < 1e-12
                else:
                    assert kth[b, g, 64 * c] == -np.inf
