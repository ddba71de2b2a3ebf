"""Pins of the oracle's query-block-granular selection (one selection per KV group and query block
of 64 tokens, the variant listed next to the per-token selection).  CPU only.

* by linearity of the score in q it is the per-token selection (pinned in test_oracle_sparse.py)
  of a query tensor whose every token holds its block's per-head sum; checked over shapes with a
  partial last block, several heads per group, batch 2, k = 0 and k above the candidate count;
* the block sum itself against hand sums;
* every token of a block receives the same row;
* a planted block whose key mean points along the block's query sum is chosen as soon as it is a
  candidate.
"""
import numpy as np
import pytest

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("B,H,Hkv,N,d,topk,n_init,n_local", [
    (1, 4, 2, 300, 16, 2, 1, 1), (2, 8, 2, 64 * 9, 8, 3, 1, 2), (1, 2, 1, 64 * 5 + 1, 4, 0, 1, 2),
    (1, 6, 3, 64 * 7 + 40, 8, 50, 1, 2)])
def test_qblock_select_is_token_selection_of_block_sums(B, H, Hkv, N, d, topk, n_init, n_local):
    q = _rand((B, H, N, d), N)
    kbar = _rand((B, Hkv, N // 64, d), N + 1)
    i1, k1 = oracle.block_select_qblock(q, kbar, 64, topk, n_init, n_local)
    i2, k2 = oracle.block_select(oracle.qblock_sum(q, 64), kbar, 64, topk, n_init, n_local)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_allclose(k1, k2, rtol=1e-12)
    for r0 in range(0, N, 64):   # one row per query block
        assert (i1[:, :, r0:r0 + 64] == i1[:, :, r0:r0 + 1]).all()


def test_qblock_sum_by_hand():
    q = np.zeros((1, 1, 130, 2))
    q[0, 0, :64, 0] = 1.0             # block 0: 64 ones in column 0
    q[0, 0, 64:128, 1] = np.arange(64)  # block 1: 0 + 1 + ... + 63 = 2016 in column 1
    q[0, 0, 128:, :] = 5.0            # partial block 2: two rows of 5
    s = oracle.qblock_sum(q, 64)
    np.testing.assert_array_equal(s[0, 0, 10], [64.0, 0.0])
    np.testing.assert_array_equal(s[0, 0, 100], [0.0, 2016.0])
    np.testing.assert_array_equal(s[0, 0, 129], [10.0, 10.0])


def test_qblock_planted_block_is_chosen():
    N, d, topk = 64 * 12, 8, 1
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 2, N, d)) * 0.01
    q[..., 0] += 1.0                      # every query block's sum points along axis 0
    kbar = rng.standard_normal((1, 1, N // 64, d)) * 0.01
    kbar[0, 0, 5, 0] = 10.0               # block 5 stands out along axis 0
    idx, _ = oracle.block_select_qblock(q, kbar, 64, topk, 1, 2)
    for c in range(N // 64):
        row = idx[0, 0, 64 * c]
        if c - 2 >= 5:                    # block 5 is a candidate (c - n_local >= 5)
            assert 5 in row, (c, row)
