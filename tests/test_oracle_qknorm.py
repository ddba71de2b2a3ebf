"""Pins of the oracle's QK normalisation (weight-free RMS norm of each head row).  CPU only.

* hand-worked rows: [3, 4] -> [3, 4] / sqrt(12.5); a one-hot row of height 2 in d = 4 keeps its
  value (its RMS is 1); these fail a sum in place of a mean;
* closed form: a constant row c of any length maps to c / sqrt(c^2 + eps), which fails eps
  added outside the square root or scaled by d;
* library routine: torch's functional rms_norm without a weight, in fp64;
* invariants with eps = 0: mean square 1, scale invariance, odd symmetry, column permutations
  commute; every row of a [B, H, N, d] tensor uses its own norm (a wrong axis fails);
* a zero row with eps > 0 stays zero (no 0/0).
"""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_hand_rows():
    got = oracle.qk_norm(np.array([[3.0, 4.0]]), eps=0.0)
    np.testing.assert_allclose(got, [[3.0 / np.sqrt(12.5), 4.0 / np.sqrt(12.5)]], rtol=1e-15)
    np.testing.assert_allclose(got, [[0.848528137423857, 1.131370849898476]], rtol=1e-14)
    got = oracle.qk_norm(np.array([[0.0, 2.0, 0.0, 0.0]]), eps=0.0)
    np.testing.assert_allclose(got, [[0.0, 2.0, 0.0, 0.0]], rtol=1e-15)


@pytest.mark.parametrize("d", [1, 2, 64, 128])
@pytest.mark.parametrize("c,eps", [(0.5, 1e-6), (-3.0, 0.25), (1e-3, 1e-6)])
def test_constant_row_closed_form(d, c, eps):
    got = oracle.qk_norm(np.full((1, d), c), eps=eps)
    np.testing.assert_allclose(got, np.full((1, d), c / np.sqrt(c * c + eps)), rtol=1e-14)


@pytest.mark.parametrize("d,eps", [(64, 1e-6), (128, 1e-5), (128, 0.0)])
def test_matches_library_rms_norm(d, eps):
    x = _rand((2, 4, 9, d), 3) * 0.7
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (d,), weight=None, eps=eps).numpy()
    np.testing.assert_allclose(oracle.qk_norm(x, eps=eps), ref, rtol=1e-13, atol=1e-15)


def test_invariants_without_eps():
    x = _rand((3, 2, 7, 128), 5) * 4.0
    y = oracle.qk_norm(x, eps=0.0)
    np.testing.assert_allclose((y * y).mean(axis=-1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(oracle.qk_norm(x * 37.5, eps=0.0), y, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(oracle.qk_norm(-x, eps=0.0), -y, rtol=0, atol=0)
    perm = np.random.default_rng(9).permutation(128)
    np.testing.assert_allclose(oracle.qk_norm(x[..., perm], eps=0.0), y[..., perm], rtol=1e-13)


def test_rows_use_their_own_norm():
    x = _rand((2, 3, 4, 64), 7)
    x[1, 2, 3] *= 1000.0
    x[0, 0, 0] *= 1e-3
    y = oracle.qk_norm(x, eps=1e-6)
    rms = np.sqrt((x * x).mean(axis=-1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(y, x / rms, rtol=1e-13)
    # the input is left untouched (the oracle returns a copy)
    assert np.abs(x[1, 2, 3]).max() > 100.0


def test_zero_row_stays_zero():
    y = oracle.qk_norm(np.zeros((2, 128)), eps=1e-6)
    assert np.all(y == 0.0)
