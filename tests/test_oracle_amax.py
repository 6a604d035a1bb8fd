"""Pins of the oracle's Amax Gain Magnitude (amax_gain) of composite residual maps.

The slavadubrov.com article prints the gain of its numpy demo (60 random 4x4 maps
I + 0.3 N(0,1), seed 0): 1906.8 for the raw product and 1.0 after Sinkhorn; its demo takes
the larger of the row and column measures.  Identity and permutation maps have gain 1
exactly, doubly stochastic maps keep every row and column sum at 1, and the first prefix
of a single map is that map's own row / column sums."""
import numpy as np

import oracle


def _stack(maps, n):
    """Layers' coefficient rows [L, 1, m] with the given H_res blocks (pre/post zero)."""
    m = n * n + 2 * n
    Hs = np.zeros((len(maps), 1, m))
    for l, A in enumerate(maps):
        Hs[l, 0, n:n + n * n] = np.asarray(A).reshape(-1)
    return Hs


def test_numpy_demo_values_printed_on_the_page():
    rng = np.random.default_rng(0)
    n, layers = 4, 60
    raw, sk = [], []
    for _ in range(layers):
        a = np.eye(n) + 0.3 * rng.standard_normal((n, n))
        raw.append(a)
        sk.append(oracle.sinkhorn(a, 20))
    g_raw = oracle.amax_gain(_stack(raw, n))[-1, 0]
    g_sk = oracle.amax_gain(_stack(sk, n))[-1, 0]
    assert f"{max(g_raw):.1f}" == "1906.8"
    assert f"{max(g_sk):.1f}" == "1.0"


def test_identity_and_permutations_have_gain_one():
    n = 5
    rng = np.random.default_rng(1)
    maps = [np.eye(n)] + [np.eye(n)[rng.permutation(n)] for _ in range(7)]
    g = oracle.amax_gain(_stack(maps, n))
    assert np.all(g == 1.0)


def test_doubly_stochastic_products_keep_gain_one():
    n = 4
    rng = np.random.default_rng(2)
    maps = [oracle.sinkhorn(rng.normal(size=(n, n)), 2000) for _ in range(30)]
    g = oracle.amax_gain(_stack(maps, n))
    assert np.abs(g - 1.0).max() < 1e-9


def test_first_prefix_is_the_map_itself_and_products_compose():
    n = 3
    rng = np.random.default_rng(3)
    A, B = rng.normal(size=(n, n)), rng.normal(size=(n, n))
    g = oracle.amax_gain(_stack([A, B], n))[:, 0]
    assert np.isclose(g[0, 0], np.abs(A).sum(axis=1).max(), rtol=1e-15)
    assert np.isclose(g[0, 1], np.abs(A).sum(axis=0).max(), rtol=1e-15)
    C = B @ A                                   # layer 2 applied after layer 1
    assert np.isclose(g[1, 0], np.abs(C).sum(axis=1).max(), rtol=1e-13)
    assert np.isclose(g[1, 1], np.abs(C).sum(axis=0).max(), rtol=1e-13)
