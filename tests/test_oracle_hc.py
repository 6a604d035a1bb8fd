"""Pins of the oracle's HC pre stage (oracle.hc_pre): the unconstrained maps the mHC pages
compare against -- a static bias plus an input-dependent term through tanh, with the same
RMSNorm and projection as mHC (slavadubrov.com article, "Kernmechanismen" and "Details van
de parameterisatie").

Each pin is fixed by the definition or by mathematics, not by retyping the oracle:
  * alpha = 0: every map is its bias, independent of X (closed form);
  * n = 1, d = 4 by hand: r = sqrt(mean x^2), one phi column per map picks one coordinate
    of x_hat (catches sum vs mean, x_hat vs X, the [pre | res | post] column order and a
    swapped bias / alpha);
  * tanh is odd: H(phi) + H(-phi) = 2 b exactly up to rounding;
  * saturation: phi scaled by 1e8 gives H = b + alpha sign(h);
  * no constraint: entries take either sign and H_res rows do not sum to 1 (a sigmoid,
    exp or Sinkhorn step left in would fail these);
  * scale invariance of the RMSNorm: H(c X) = H(X) for c > 0.
"""
import math

import numpy as np

import oracle


def _rand(n, d, T=7, seed=0):
    rng = np.random.default_rng(seed)
    m = n * n + 2 * n
    X = rng.standard_normal((T, n, d))
    phi = rng.standard_normal((n * d, m)) / math.sqrt(n * d)
    b_pre, b_post = rng.standard_normal(n) * 0.3, rng.standard_normal(n) * 0.3
    b_res = np.eye(n) + rng.standard_normal((n, n)) * 0.1
    return X, phi, b_pre, b_post, b_res


def test_alpha_zero_gives_the_biases():
    X, phi, bp, bq, br = _rand(4, 16)
    x_in, H = oracle.hc_pre(X, phi, bp, bq, br, 0.0, 0.0, 0.0)
    expect = np.concatenate([bp, br.reshape(-1), bq])
    assert np.array_equal(H, np.broadcast_to(expect, H.shape))
    assert np.allclose(x_in, np.einsum("i,tic->tc", bp, X), rtol=0, atol=1e-14)


def test_n1_by_hand():
    X = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    phi = np.zeros((4, 3))
    phi[0, 0] = 1.0          # pre  <- x_hat[0]
    phi[1, 1] = 1.0          # res  <- x_hat[1]
    phi[3, 2] = 1.0          # post <- x_hat[3]
    r = math.sqrt((1 + 4 + 9 + 16) / 4.0)
    x_in, H = oracle.hc_pre(X, phi, [0.5], [-0.25], [[1.0]], 0.3, 0.1, 0.2, eps=0.0)
    hp = 0.5 + 0.3 * math.tanh(1.0 / r)
    hr = 1.0 + 0.2 * math.tanh(2.0 / r)
    hq = -0.25 + 0.1 * math.tanh(4.0 / r)
    assert np.allclose(H[0], [hp, hr, hq], rtol=0, atol=1e-15)
    assert np.allclose(x_in[0], hp * X[0, 0], rtol=0, atol=1e-14)


def test_tanh_is_odd():
    X, phi, bp, bq, br = _rand(3, 24, seed=1)
    a = (0.7, 0.4, 0.9)
    _, H1 = oracle.hc_pre(X, phi, bp, bq, br, *a)
    _, H2 = oracle.hc_pre(X, -phi, bp, bq, br, *a)
    b = np.concatenate([bp, br.reshape(-1), bq])
    assert np.allclose(H1 + H2, 2 * b, rtol=0, atol=1e-14)
    assert not np.allclose(H1, H2)


def test_saturation():
    X, phi, bp, bq, br = _rand(4, 8, seed=2)
    a = (0.5, 0.25, 2.0)
    _, H = oracle.hc_pre(X, phi * 1e8, bp, bq, br, *a)
    h = oracle.mhc_projection(X, phi)
    n = 4
    alpha = np.concatenate([np.full(n, a[0]), np.full(n * n, a[2]), np.full(n, a[1])])
    b = np.concatenate([bp, br.reshape(-1), bq])
    assert np.allclose(H, b + alpha * np.sign(h), rtol=0, atol=1e-14)


def test_unconstrained_signs_and_rows():
    X, phi, _, _, _ = _rand(4, 32, T=64, seed=3)
    z = np.zeros(4)
    _, H = oracle.hc_pre(X, phi, z, z, np.zeros((4, 4)), 1.0, 1.0, 1.0)
    Hp, Hr, Hq = oracle.split_H(H, 4)
    assert (Hp < 0).any() and (Hp > 0).any()
    assert (Hr < 0).any() and (Hq < 0).any()
    assert np.abs(Hr.sum(axis=2) - 1).max() > 1e-2


def test_scale_invariance():
    X, phi, bp, bq, br = _rand(2, 40, seed=4)
    _, H1 = oracle.hc_pre(X, phi, bp, bq, br, 0.5, 0.5, 0.5)
    _, H2 = oracle.hc_pre(X * 37.5, phi, bp, bq, br, 0.5, 0.5, 0.5)
    assert np.allclose(H1, H2, rtol=0, atol=1e-14)


def test_threads_do_not_change_results():
    X, phi, bp, bq, br = _rand(4, 64, T=40, seed=5)
    a1 = oracle.hc_pre(X, phi, bp, bq, br, 0.3, 0.2, 0.1, nthreads=1)
    a4 = oracle.hc_pre(X, phi, bp, bq, br, 0.3, 0.2, 0.1, nthreads=4)
    assert np.array_equal(a1[0], a4[0]) and np.array_equal(a1[1], a4[1])
