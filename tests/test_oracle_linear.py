"""Pins for the oracle's linear (Lightning-style) attention.

The pages print no worked example, so the oracle is pinned by mathematics it must satisfy:

* three independent statements of the definition (recurrent, quadratic, chunked at several
  chunk sizes) agree to ~1e-12;                                           [invariant]
* lambda = 1 is plain causal linear attention, a cumulative sum of k^T v; [closed form]
* lambda = 0 keeps only the diagonal term (q_i.k_i) v_i;                   [closed form]
* a scalar case worked by hand (tests/golden/linear_scalar.json);         [closed form]
* prefill split at any point and resumed from the carried state equals one prefill, and decode
  steps reproduce prefill rows and the final state.                       [invariant]

A dropped term (the carried state), an off-by-one decay exponent, or a transposed state
(v^T k instead of k^T v, with d_k != d_v) each fails at least one of these.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def _inputs(rng, B=2, H=3, N=37, dk=5, dv=4, lam=None):
    q = _rand((B, H, N, dk), rng, 0.5)
    k = _rand((B, H, N, dk), rng, 0.5)
    v = _rand((B, H, N, dv), rng)
    if lam is None:
        lam = rng.uniform(0.3, 1.0, size=H)
    return q, k, v, np.asarray(lam, dtype=np.float64)


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


def test_three_forms_agree():
    rng = np.random.default_rng(1)
    q, k, v, lam = _inputs(rng)
    o_rec, s_rec = oracle.linear_recurrent(q, k, v, lam)
    o_quad = oracle.linear_quadratic(q, k, v, lam)
    assert _rel(o_quad, o_rec) < 1e-12
    for C in (1, 4, 16, 64):
        o_ch, s_ch = oracle.linear_chunked(q, k, v, lam, C)
        assert _rel(o_ch, o_rec) < 1e-12, C
        assert _rel(s_ch, s_rec) < 1e-12, C


def test_three_forms_agree_with_state_in():
    rng = np.random.default_rng(2)
    q, k, v, lam = _inputs(rng, N=29)
    s0 = _rand((2, 3, 5, 4), rng)
    o_rec, s_rec = oracle.linear_recurrent(q, k, v, lam, s0)
    o_quad = oracle.linear_quadratic(q, k, v, lam, s0)
    o_ch, s_ch = oracle.linear_chunked(q, k, v, lam, 8, s0)
    assert _rel(o_quad, o_rec) < 1e-12
    assert _rel(o_ch, o_rec) < 1e-12
    assert _rel(s_ch, s_rec) < 1e-12


def test_lambda_one_is_cumulative_sum():
    # Causal linear attention without decay: o_i = q_i (sum_{j<=i} k_j^T v_j).
    rng = np.random.default_rng(3)
    q, k, v, _ = _inputs(rng, B=1, H=2, N=20, dk=3, dv=6)
    lam = np.ones(2)
    outer = np.einsum("bhna,bhnc->bhnac", k, v)
    S = np.cumsum(outer, axis=2)
    expect = np.einsum("bhna,bhnac->bhnc", q, S)
    for o in (oracle.linear_recurrent(q, k, v, lam)[0], oracle.linear_quadratic(q, k, v, lam),
              oracle.linear_chunked(q, k, v, lam, 7)[0]):
        assert _rel(o, expect) < 1e-12


def test_lambda_zero_keeps_diagonal():
    # 0^0 = 1: only j = i survives.
    rng = np.random.default_rng(4)
    q, k, v, _ = _inputs(rng, B=1, H=1, N=11, dk=4, dv=3)
    lam = np.zeros(1)
    expect = np.einsum("bhna,bhna->bhn", q, k)[..., None] * v
    for o in (oracle.linear_recurrent(q, k, v, lam)[0], oracle.linear_quadratic(q, k, v, lam),
              oracle.linear_chunked(q, k, v, lam, 4)[0]):
        assert _rel(o, expect) < 1e-13


def test_scalar_worked_example():
    g = json.load(open(os.path.join(GOLD, "linear_scalar.json")))
    q = np.array(g["q"], float).reshape(1, 1, -1, 1)
    k = np.array(g["k"], float).reshape(1, 1, -1, 1)
    v = np.array(g["v"], float).reshape(1, 1, -1, 1)
    lam = np.array([g["lam"]])
    for case in g["cases"]:
        s0 = np.full((1, 1, 1, 1), float(case["S_in"]))
        o, s = oracle.linear_recurrent(q, k, v, lam, s0)
        np.testing.assert_allclose(o.ravel(), case["o"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(s.ravel(), [case["S_out"]], rtol=0, atol=1e-14)
        oq = oracle.linear_quadratic(q, k, v, lam, s0)
        np.testing.assert_allclose(oq.ravel(), case["o"], rtol=0, atol=1e-14)
        oc, sc = oracle.linear_chunked(q, k, v, lam, 2, s0)
        np.testing.assert_allclose(oc.ravel(), case["o"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(sc.ravel(), [case["S_out"]], rtol=0, atol=1e-14)


@pytest.mark.parametrize("split", [1, 13, 31])
def test_split_and_resume(split):
    rng = np.random.default_rng(5)
    q, k, v, lam = _inputs(rng, N=32)
    o_full, s_full = oracle.linear_chunked(q, k, v, lam, 8)
    o1, s1 = oracle.linear_chunked(q[:, :, :split], k[:, :, :split], v[:, :, :split], lam, 8)
    o2, s2 = oracle.linear_chunked(q[:, :, split:], k[:, :, split:], v[:, :, split:], lam, 8, s1)
    assert _rel(np.concatenate([o1, o2], axis=2), o_full) < 1e-12
    assert _rel(s2, s_full) < 1e-12


def test_decode_reproduces_prefill():
    rng = np.random.default_rng(6)
    q, k, v, lam = _inputs(rng, N=9)
    o_pre, s_pre = oracle.linear_recurrent(q, k, v, lam)
    S = np.zeros((2, 3, 5, 4))
    for i in range(9):
        o, S = oracle.linear_decode(q[:, :, i], k[:, :, i], v[:, :, i], lam, S)
        assert _rel(o, o_pre[:, :, i]) < 1e-12
    assert _rel(S, s_pre) < 1e-12


def test_quadratic_rows_subset():
    rng = np.random.default_rng(7)
    q, k, v, lam = _inputs(rng)
    s0 = _rand((2, 3, 5, 4), rng)
    full = oracle.linear_quadratic(q, k, v, lam, s0)
    rows = np.array([[0, 0], [5, 36], [3, 17], [2, 1]])
    sub = oracle.linear_quadratic(q, k, v, lam, s0, rows=rows)
    B, H = 2, 3
    for n, (bh, i) in enumerate(rows):
        np.testing.assert_array_equal(sub[n], full[bh // H, bh % H, i])


def test_deep_decay_stays_finite():
    # lambda = 0.431 (the fastest decay of the 32-head recipe) over 300 steps: exponents up to
    # 299 underflow gracefully to 0 and never produce inf/nan.
    rng = np.random.default_rng(8)
    q, k, v, _ = _inputs(rng, B=1, H=1, N=300, dk=4, dv=4)
    lam = np.array([np.exp(-2 ** -0.25)])
    o, s = oracle.linear_chunked(q, k, v, lam, 64)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(s))
    assert _rel(o, oracle.linear_recurrent(q, k, v, lam)[0]) < 1e-12
