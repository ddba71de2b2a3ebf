"""Pins of the oracle's backward pass of the linear attention (gradients of sum(o * do) with respect
to q, k, v for a fresh sequence).  CPU only.

* central finite differences of the pinned forward (oracle.linear_quadratic) at every element of
  q, k and v on a small case with two heads and different decays;
* lam = 0: o_i = (q_i . k_i) v_i, whose gradients are written out here element-wise
  (dq_i = (do_i . v_i) k_i, dk_i = (do_i . v_i) q_i, dv_i = (q_i . k_i) do_i).
"""
import numpy as np

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_linear_backward_finite_differences():
    B, H, N, d = 1, 2, 6, 3
    q, k, v, do = (_rand((B, H, N, d), s) for s in (1, 2, 3, 4))
    lam = np.array([0.8, 0.95])
    dq, dk, dv = oracle.linear_backward(q, k, v, lam, do)
    f = lambda q_, k_, v_: float(np.sum(oracle.linear_quadratic(q_, k_, v_, lam) * do))
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for ix in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[ix] += h
            xm[ix] -= h
            args_p = [xp if name == n else y for n, y in (("q", q), ("k", k), ("v", v))]
            args_m = [xm if name == n else y for n, y in (("q", q), ("k", k), ("v", v))]
            num[ix] = (f(*args_p) - f(*args_m)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_linear_backward_zero_decay_closed_form():
    B, H, N, d = 1, 1, 5, 4
    q, k, v, do = (_rand((B, H, N, d), s) for s in (5, 6, 7, 8))
    dq, dk, dv = oracle.linear_backward(q, k, v, np.array([0.0]), do)
    dov = np.sum(do * v, axis=-1, keepdims=True)
    qk = np.sum(q * k, axis=-1, keepdims=True)
    np.testing.assert_allclose(dq, dov * k, atol=1e-12)
    np.testing.assert_allclose(dk, dov * q, atol=1e-12)
    np.testing.assert_allclose(dv, qk * do, atol=1e-12)
