"""Pins for the fp64 oracle: values the pages print, closed forms and invariants.

Each test names the passage it checks.  Together they are chosen so that a plausible
mistake in the oracle -- rows normalised before columns, a missing exp, a wrong flatten
index, a transposed H_res, sigma and 2*sigma swapped, sum instead of mean in RMSNorm,
x_hat instead of raw X in the read map, a wrong phi column order, an off-by-one in the
Sinkhorn loop -- fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle
from mhc_hyper_connections_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    blocks, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                cur = line.strip("[]")
                blocks[cur] = []
            else:
                blocks[cur].append([float(v) for v in line.split()])
    return {k: np.array(v) for k, v in blocks.items()}


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


# ---------------------------------------------------------------- Sinkhorn-Knopp

def test_sinkhorn_worked_example_3x3():
    """slavadubrov.com mHC article, "Sinkhorn-Knopp-projectie": the printed 3x3 example
    (exp, one pass with column sums 1.030/1.092/0.877, twenty passes), 3 decimals.
    Pins the exp, the column-then-row order and the per-pass step."""
    g = _read_golden("sinkhorn_3x3.txt")
    A = g["logits"]
    tol = 5e-4 + 1e-9
    np.testing.assert_allclose(oracle.sinkhorn(A, 0), g["exp"], atol=tol, rtol=0)
    S1 = oracle.sinkhorn(A, 1)
    np.testing.assert_allclose(S1, g["pass1"], atol=tol, rtol=0)
    np.testing.assert_allclose(S1.sum(axis=1), g["pass1_row_sums"][0], atol=tol, rtol=0)
    np.testing.assert_allclose(S1.sum(axis=0), g["pass1_col_sums"][0], atol=tol, rtol=0)
    S20 = oracle.sinkhorn(A, 20)
    np.testing.assert_allclose(S20, g["pass20"], atol=tol, rtol=0)
    np.testing.assert_allclose(S20.sum(axis=0), g["pass20_col_sums"][0], atol=tol, rtol=0)
    # the page: after one pass the largest column deviation is about 12 %
    assert abs(np.abs(S1.sum(axis=0) - 1).max() - 0.123) < 1e-3
    # rows-first would give different one-pass values: the pin is discriminating
    M = np.exp(A)
    M = M / M.sum(axis=1, keepdims=True)
    M = M / M.sum(axis=0, keepdims=True)
    assert np.abs(M - g["pass1"]).max() > 0.01


def test_sinkhorn_numpy_demo_amax():
    """slavadubrov.com mHC article, the NumPy demo after the 3x3 example: seed 0, 60
    random 4x4 maps I + 0.3 N(0,1); the page prints Amax 1906.8 for the raw product and
    1.0 for the product of Sinkhorn-projected maps (20 iterations)."""
    rng = np.random.default_rng(0)
    n, layers = 4, 60
    hc, mhc = np.eye(n), np.eye(n)
    for _ in range(layers):
        a = np.eye(n) + 0.3 * rng.standard_normal((n, n))
        hc = a @ hc
        mhc = oracle.sinkhorn(a, 20) @ mhc

    def amax(m):  # max absolute row sum / column sum ("Amax Gain Magnitude")
        return max(np.abs(m).sum(axis=1).max(), np.abs(m).sum(axis=0).max())

    assert f"{amax(hc):.1f}" == "1906.8"
    assert f"{amax(mhc):.1f}" == "1.0"


def test_sinkhorn_t0_is_exp_and_t1_closed_form():
    """t_max = 0 is M0 = exp(B~) ("DeepSeek-V4/mhc", equation sinkhorn-init); one round
    is T_r(T_c(M0)) written out with math.exp and explicit sums."""
    rng = np.random.default_rng(5)
    L = rng.standard_normal((3, 3))
    E = np.array([[math.exp(L[i, j]) for j in range(3)] for i in range(3)])
    np.testing.assert_array_equal(oracle.sinkhorn(L, 0), E)
    C = np.array([[E[i, j] / sum(E[k, j] for k in range(3)) for j in range(3)] for i in range(3)])
    R = np.array([[C[i, j] / sum(C[i, k] for k in range(3)) for j in range(3)] for i in range(3)])
    np.testing.assert_allclose(oracle.sinkhorn(L, 1), R, rtol=1e-15, atol=0)


@pytest.mark.parametrize("n", [2, 3, 4, 8])
def test_sinkhorn_invariants(n):
    """Birkhoff properties on the knowledge page ("mHC 的流形约束怎么保稳定"): entries
    non-negative; after the final row step every row sums to 1; the column error shrinks
    with t; ||H||_2 <= sqrt(||H||_1 ||H||_inf) (the bound the page quotes) and -> 1."""
    rng = np.random.default_rng(100 + n)
    for _ in range(50):
        L = 4 * np.eye(n) + rng.standard_normal((n, n)) * math.sqrt(0.1)
        L = L + 0.01 * rng.standard_normal((n, n))
        H = oracle.sinkhorn(L, 20)
        assert (H > 0).all()
        assert np.abs(H.sum(axis=1) - 1).max() <= 8 * n * np.finfo(float).eps
        errs = [np.abs(oracle.sinkhorn(L, t).sum(axis=0) - 1).max() for t in (1, 2, 5, 10, 20)]
        assert all(b <= a * (1 + 1e-12) for a, b in zip(errs, errs[1:]))
        assert errs[-1] <= 1e-2
        s2 = np.linalg.norm(H, 2)
        assert s2 <= math.sqrt(np.abs(H).sum(axis=0).max() * np.abs(H).sum(axis=1).max()) * (1 + 1e-12)
        # converges to doubly stochastic (slow for near-diagonal 2x2 maps: use many rounds)
        Hinf = oracle.sinkhorn(L, 1000)
        assert np.abs(Hinf.sum(axis=0) - 1).max() <= 1e-12
        assert np.linalg.norm(Hinf, 2) <= 1 + 1e-12


def test_sinkhorn_circulant_closed_form():
    """A circulant exp(L) has equal row and column sums, so the first column step already
    makes it doubly stochastic: H = exp(L) / rowsum(exp(L)) for every t >= 1."""
    c = np.array([0.3, -1.2, 2.0, 0.7])
    L = np.array([[c[(j - i) % 4] for j in range(4)] for i in range(4)])
    E = np.exp(L)
    expect = E / E[0].sum()
    for t in (1, 3, 20):
        np.testing.assert_allclose(oracle.sinkhorn(L, t), expect, rtol=1e-14, atol=0)


def test_sinkhorn_permutation_limit():
    """Large logits on a permutation converge to that permutation matrix (Birkhoff-von
    Neumann vertices, slavadubrov.com article "Wat doubly stochastic garandeert")."""
    P = np.zeros((4, 4))
    for i, j in enumerate([2, 0, 3, 1]):
        P[i, j] = 1
    H = oracle.sinkhorn(40 * P, 20)
    np.testing.assert_allclose(H, P, atol=1e-12)


# ---------------------------------------------------------------- pre stage

def _pre(X, phi, b_pre, b_post, b_res, a=(0.01, 0.01, 0.01), eps=1e-20, t_max=20):
    return oracle.mhc_pre(X, phi, b_pre, b_post, b_res, a[0], a[1], a[2], eps=eps, t_max=t_max)


def test_alpha_zero_gives_bias_only_maps():
    """"DeepSeek-V4/mhc", equations a/b/c-tilde: with alpha = 0 the maps are the static
    biases only, independent of X; 2*sigmoid(0) = 1 (slavadubrov.com, "Details van de
    parameterisatie")."""
    w = wl.make_inputs(T=5, n=4, d=16, dtype="f32", seed=7)
    X = w.values(w.X)
    b_pre = np.array([0.0, 1.0, -2.0, 0.5])
    b_post = np.array([0.0, -1.0, 3.0, 0.25])
    x_in, H = _pre(X, w.phi, b_pre, b_post, w.b_res, a=(0, 0, 0))
    Hp, Hr, Hq = oracle.split_H(H, 4)
    for t in range(5):
        for i in range(4):
            assert Hp[t, i] == pytest.approx(_sig(b_pre[i]), rel=1e-15)
            assert Hq[t, i] == pytest.approx(2 * _sig(b_post[i]), rel=1e-15)
        np.testing.assert_allclose(Hr[t], oracle.sinkhorn(w.b_res, 20), rtol=1e-15)
    assert Hp[0, 0] == 0.5 and Hq[0, 0] == 1.0
    # read map on raw X
    np.testing.assert_allclose(x_in, np.einsum("i,tic->tc", Hp[0], X), rtol=1e-13, atol=1e-14)


def test_n1_closed_form_by_hand():
    """n = 1, d = 4, X = [1, 2, 3, 4]: RMSNorm over n*d with eps inside the root (mean of
    squares = 7.5); H_res of a 1x1 map is 1; x_in = H_pre X on raw X; X' = X + H_post F
    (slavadubrov.com Eq. 3 reduces to the standard residual at n = 1 with unit maps)."""
    X = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    F = np.array([[0.5, -1.0, 2.0, 0.0]])
    phi = np.zeros((4, 3))
    phi[2, 0] = 1.0              # pre column picks x_hat[2] = 3 / r
    phi[:, 1] = 5.0              # res column: irrelevant, H_res = 1 for n = 1
    phi[:, 2] = 1.0              # post column: sum of x_hat = 10 / r
    a_pre, a_res, a_post = 0.3, 0.7, -0.2
    b_pre, b_post, b_res = 0.1, -0.4, 0.9
    x_in, H = oracle.mhc_pre(X, phi, [b_pre], [b_post], [[b_res]], a_pre, a_post, a_res,
                             eps=1e-20, t_max=20)
    r = math.sqrt(30.0 / 4.0 + 1e-20)
    hp = _sig(a_pre * 3.0 / r + b_pre)
    hq = 2 * _sig(a_post * 10.0 / r + b_post)
    assert H[0, 0] == pytest.approx(hp, rel=1e-15)
    assert H[0, 1] == 1.0
    assert H[0, 2] == pytest.approx(hq, rel=1e-15)
    np.testing.assert_allclose(x_in[0], hp * X[0, 0], rtol=1e-15)
    out = oracle.mhc_post(X, F, H)
    np.testing.assert_allclose(out[0, 0], X[0, 0] + hq * F[0], rtol=1e-15)
    # standard residual: zero biases, alpha = 0 -> X' = X + F
    _, H0 = oracle.mhc_pre(X, phi, [0.0], [0.0], [[0.0]], 0, 0, 0)
    np.testing.assert_array_equal(oracle.mhc_post(X, F, H0)[0, 0], X[0, 0] + F[0])


def test_flatten_index_is_stream_major():
    """vec(X) is the row-stacked flatten of the n x d stream matrix (element (i, c) at
    i*d + c; "DeepSeek-V4/mhc", HC section: row i is stream i).  A phi with one non-zero
    entry at row k makes h_pre,0 = x_hat[k]."""
    n, d = 2, 3
    rng = np.random.default_rng(11)
    X = rng.standard_normal((1, n, d))
    r = math.sqrt((X ** 2).mean() + 1e-20)
    for i in range(n):
        for c in range(d):
            phi = np.zeros((n * d, n * n + 2 * n))
            phi[i * d + c, 0] = 1.0
            _, H = _pre(X, phi, np.zeros(n), np.zeros(n), np.zeros((n, n)), a=(1.0, 1.0, 1.0))
            assert H[0, 0] == pytest.approx(_sig(X[0, i, c] / r), rel=1e-14)
            assert H[0, 1] == 0.5


def test_phi_column_order_pre_res_post():
    """phi columns are [pre (n) | res (n^2, row-major Mat) | post (n)] ("DeepSeek-V4/mhc",
    the 4 + 16 + 4 = 24 output columns of the thin GEMM).  A phi that is non-zero in one
    column moves only the map that column feeds."""
    n, d = 3, 4
    m = n * n + 2 * n
    rng = np.random.default_rng(12)
    X = rng.standard_normal((2, n, d))
    b_res = 2 * np.eye(n) + 0.3 * rng.standard_normal((n, n))
    base_x, base_H = _pre(X, np.zeros((n * d, m)), np.zeros(n), np.zeros(n), b_res)
    for j in range(m):
        phi = np.zeros((n * d, m))
        phi[:, j] = rng.standard_normal(n * d)
        _, H = _pre(X, phi, np.zeros(n), np.zeros(n), b_res, a=(1.0, 1.0, 1.0))
        moved = np.abs(H - base_H).max(axis=0) > 1e-12
        if j < n:
            assert moved.tolist() == [k == j for k in range(m)]
        elif j < n + n * n:
            assert not moved[:n].any() and not moved[n + n * n:].any() and moved[n:n + n * n].any()
            # Mat is row-major: entry (i, k) of the logits is h[n + i*n + k]
            i, k = divmod(j - n, n)
            for t in range(2):
                xh = X[t].reshape(-1) / math.sqrt((X[t] ** 2).mean() + 1e-20)
                L = b_res.copy()
                L[i, k] += xh @ phi[:, j]
                np.testing.assert_allclose(H[t, n:n + n * n].reshape(n, n),
                                           oracle.sinkhorn(L, 20), rtol=1e-13, atol=1e-15)
        else:
            assert moved.tolist() == [k == j for k in range(m)]


def test_rmsnorm_scale_invariance():
    """x_hat = RMSNorm(vec X) is invariant to X -> cX (c > 0, eps negligible), so H is,
    and the read map on raw X scales with c."""
    w = wl.make_inputs(T=6, n=4, d=32, dtype="f32", seed=13, alpha=0.5)
    X = w.values(w.X)
    x1, H1 = _pre(X, w.phi, w.b_pre, w.b_post, w.b_res, a=(0.5, 0.5, 0.5))
    x2, H2 = _pre(7.5 * X, w.phi, w.b_pre, w.b_post, w.b_res, a=(0.5, 0.5, 0.5))
    np.testing.assert_allclose(H2, H1, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(x2, 7.5 * x1, rtol=1e-13, atol=1e-13)


def test_stream_permutation_equivariance():
    """Relabelling the streams (X rows, phi row blocks and columns, biases) relabels the
    maps: H_pre -> H_pre[s], H_res -> H_res[s][:, s], H_post -> H_post[s]; x_in and the
    post output follow."""
    n, d = 4, 8
    w = wl.make_inputs(T=3, n=n, d=d, dtype="f32", seed=14, alpha=0.7)
    X = w.values(w.X)
    b_pre = np.array([0.1, -0.3, 0.2, 0.0])
    b_post = np.array([-0.2, 0.4, 0.0, 0.3])
    s = np.array([2, 0, 3, 1])
    a = (0.7, 0.7, 0.7)
    x1, H1 = _pre(X, w.phi, b_pre, b_post, w.b_res, a=a)
    rows = np.concatenate([np.arange(d) + si * d for si in s])
    cols = np.concatenate([s, n + (s[:, None] * n + s[None, :]).reshape(-1), n + n * n + s])
    phi2 = w.phi.astype(np.float64)[rows][:, cols]
    x2, H2 = _pre(X[:, s, :], phi2, b_pre[s], b_post[s], w.b_res[s][:, s], a=a)
    P1, R1, Q1 = oracle.split_H(H1, n)
    P2, R2, Q2 = oracle.split_H(H2, n)
    np.testing.assert_allclose(P2, P1[:, s], rtol=1e-13)
    np.testing.assert_allclose(Q2, Q1[:, s], rtol=1e-13)
    np.testing.assert_allclose(R2, R1[:, s][:, :, s], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(x2, x1, rtol=1e-12, atol=1e-13)
    F = w.values(w.F_out)
    np.testing.assert_allclose(oracle.mhc_post(X[:, s, :], F, H2),
                               oracle.mhc_post(X, F, H1)[:, s, :], rtol=1e-12, atol=1e-13)


def test_zero_token_gives_bias_maps():
    """An all-zero token: mean square 0, r = sqrt(eps), x_hat = 0, so the logits are the
    biases and x_in = 0."""
    w = wl.make_inputs(T=2, n=4, d=16, dtype="f32", seed=15)
    X = w.values(w.X)
    X[1] = 0.0
    x_in, H = _pre(X, w.phi, w.b_pre, w.b_post, w.b_res)
    _, Hb = _pre(X, w.phi, w.b_pre, w.b_post, w.b_res, a=(0, 0, 0))
    np.testing.assert_array_equal(H[1], Hb[1])
    assert (x_in[1] == 0).all()


# ---------------------------------------------------------------- post stage

def test_post_hand_built_maps():
    """X'_i = sum_j H_res[i][j] X_j + H_post[i] F_out (slavadubrov.com Eq. 3): with H_res a
    non-symmetric permutation, output stream i is input stream p(i) plus H_post[i] F.
    Catches a transposed H_res.  H_res = I, H_post = 0 returns X exactly."""
    n, d, T = 4, 6, 3
    rng = np.random.default_rng(16)
    X = rng.standard_normal((T, n, d))
    F = rng.standard_normal((T, d))
    p = [1, 2, 3, 0]
    P = np.zeros((n, n))
    for i, j in enumerate(p):
        P[i, j] = 1.0
    hpost = np.array([0.5, 1.0, 1.5, 2.0])
    H = np.concatenate([np.full(n, 0.5), P.reshape(-1), hpost])[None].repeat(T, 0)
    out = oracle.mhc_post(X, F, H)
    for t in range(T):
        for i in range(n):
            np.testing.assert_array_equal(out[t, i], X[t, p[i]] + hpost[i] * F[t])
    Hid = np.concatenate([np.zeros(n), np.eye(n).reshape(-1), np.zeros(n)])[None].repeat(T, 0)
    np.testing.assert_array_equal(oracle.mhc_post(X, F, Hid), X)


def test_post_is_linear_in_X_and_F():
    n, d, T = 3, 5, 4
    rng = np.random.default_rng(17)
    X1, X2 = rng.standard_normal((2, T, n, d))
    F1, F2 = rng.standard_normal((2, T, d))
    H = rng.random((T, n * n + 2 * n))
    lhs = oracle.mhc_post(2 * X1 - 3 * X2, 2 * F1 - 3 * F2, H)
    rhs = 2 * oracle.mhc_post(X1, F1, H) - 3 * oracle.mhc_post(X2, F2, H)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- whole map, cross-check

def test_tiny_against_independent_numpy_expression():
    """Cross-check at a tiny size against a vectorised numpy fp64 expression written here
    (einsum / broadcasting, not the oracle's loops)."""
    w = wl.make_inputs(T=7, n=4, d=24, dtype="f32", seed=18, alpha=0.3)
    X, F = w.values(w.X), w.values(w.F_out)
    n, T = 4, 7
    x_in, H = _pre(X, w.phi, w.b_pre, w.b_post, w.b_res, a=(0.3, 0.3, 0.3))
    v = X.reshape(T, -1)
    xh = v / np.sqrt((v ** 2).mean(axis=1, keepdims=True) + 1e-20)
    h = xh @ w.phi.astype(np.float64)
    hp = 1 / (1 + np.exp(-(0.3 * h[:, :n] + w.b_pre)))
    hq = 2 / (1 + np.exp(-(0.3 * h[:, n + n * n:] + w.b_post)))
    M = np.exp(0.3 * h[:, n:n + n * n].reshape(T, n, n) + w.b_res)
    for _ in range(20):
        M = M / M.sum(axis=1, keepdims=True)
        M = M / M.sum(axis=2, keepdims=True)
    np.testing.assert_allclose(H[:, :n], hp, rtol=1e-13)
    np.testing.assert_allclose(H[:, n + n * n:], hq, rtol=1e-13)
    np.testing.assert_allclose(H[:, n:n + n * n].reshape(T, n, n), M, rtol=1e-12)
    np.testing.assert_allclose(x_in, np.einsum("ti,tic->tc", hp, X), rtol=1e-12, atol=1e-13)
    out = oracle.mhc_post(X, F, H)
    ref = np.einsum("tij,tjc->tic", M, X) + hq[:, :, None] * F[:, None, :]
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_threads_do_not_change_results():
    w = wl.make_inputs(T=33, n=4, d=32, dtype="bf16", seed=19)
    X = w.values(w.X)
    a = oracle.mhc_pre(X, w.phi, w.b_pre, w.b_post, w.b_res, 0.01, 0.01, 0.01, nthreads=1)
    b = oracle.mhc_pre(X, w.phi, w.b_pre, w.b_post, w.b_res, 0.01, 0.01, 0.01, nthreads=4)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
