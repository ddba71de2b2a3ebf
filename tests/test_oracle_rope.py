"""Pins of the oracle's rotary position embedding (the linear layers' half of HyPE) and of the
RoPE linear attention built on it.  CPU only.

* library routine: the rotation equals the complex product (x_i + i x_{i+d/2}) e^{i p theta_i},
  with numpy's complex exponential and theta_i = base^(-2i/d); this fixes the pairing (i with
  i + d/2) and the sign of the sine;
* invariants: identity at position 0; every pair's length preserved; R(m) R(n) = R(m + n);
  <R(m) q, R(n) k> = <R(m - n) q, k> (attention scores see only relative positions);
* the RoPE linear attention of a fresh sequence does not depend on where the sequence starts
  (a shift of every position rotates q_i and k_j alike), which fails if only one of q, k is
  rotated or if the two use different positions.
"""
import numpy as np
import pytest

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("d,base", [(2, 10000.0), (8, 100.0), (128, 10000.0), (64, 500000.0)])
def test_rope_is_complex_rotation(d, base):
    x = _rand((2, 3, 5, d), 1)
    pos0 = 777
    got = oracle.rope(x, pos0, base)
    half = d // 2
    theta = base ** (-2.0 * np.arange(half) / d)
    pos = pos0 + np.arange(5)[:, None]
    z = (x[..., :half] + 1j * x[..., half:]) * np.exp(1j * pos * theta)
    np.testing.assert_allclose(got[..., :half], z.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[..., half:], z.imag, rtol=0, atol=1e-12)


def test_rope_invariants():
    d = 16
    x = _rand((1, 2, 1, d), 2)
    np.testing.assert_array_equal(oracle.rope(x, 0), x)                       # position 0
    y = oracle.rope(x, 12345)
    half = d // 2
    np.testing.assert_allclose(np.hypot(y[..., :half], y[..., half:]),
                               np.hypot(x[..., :half], x[..., half:]), rtol=1e-13)
    np.testing.assert_allclose(oracle.rope(oracle.rope(x, 40), 2), oracle.rope(x, 42), atol=1e-12)
    q, k = _rand((1, 1, 1, d), 3), _rand((1, 1, 1, d), 4)
    for m, n in [(5, 3), (1000, 999), (70000, 12)]:
        lhs = np.sum(oracle.rope(q, m) * oracle.rope(k, n))
        rhs = np.sum(oracle.rope(q, m - n) * k)
        assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(rhs)), (m, n, lhs, rhs)


def test_rope_linear_attention_is_translation_invariant():
    B, H, N, d = 1, 2, 40, 16
    q, k, v = _rand((B, H, N, d), 5), _rand((B, H, N, d), 6), _rand((B, H, N, d), 7)
    lam = np.array([0.9, 0.99])
    o0, _ = oracle.linear_chunked_rope(q, k, v, lam, 16, pos0=0)
    o1, _ = oracle.linear_chunked_rope(q, k, v, lam, 16, pos0=100003)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-9 * np.abs(o0).max())
    # and it is not the plain linear attention (the rotation does act)
    o_plain, _ = oracle.linear_chunked(q, k, v, lam, 16)
    assert np.abs(o_plain - o0).max() > 1e-3 * np.abs(o0).max()


def test_rope_linear_attention_resumes_across_a_split():
    # prefill(N1) -> state -> prefill(N2) at pos0 = N1 equals one prefill of N1 + N2 rows
    B, H, N, d = 1, 2, 50, 8
    q, k, v = _rand((B, H, N, d), 8), _rand((B, H, N, d), 9), _rand((B, H, N, d), 10)
    lam = np.array([0.95, 0.8])
    o, s = oracle.linear_chunked_rope(q, k, v, lam, 16, pos0=7)
    n1 = 23
    o_a, s_a = oracle.linear_chunked_rope(q[:, :, :n1], k[:, :, :n1], v[:, :, :n1], lam, 16, pos0=7)
    o_b, s_b = oracle.linear_chunked_rope(q[:, :, n1:], k[:, :, n1:], v[:, :, n1:], lam, 16,
                                          pos0=7 + n1, s_in=s_a)
    np.testing.assert_allclose(np.concatenate([o_a, o_b], axis=2), o, atol=1e-12 * np.abs(o).max())
    np.testing.assert_allclose(s_b, s, atol=1e-12 * np.abs(s).max())
