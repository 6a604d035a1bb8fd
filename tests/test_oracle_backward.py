"""Pins of the oracle's reverse mode (mhc_backward) against what the forward fixes.

The backward is the gradient of L = <dX_out, X'> + <dx_in, x_in> over the inputs of pre +
post.  Its pin is independent of its own code: central finite differences of the forward
oracle (itself pinned in test_oracle_pins.py) for every input element at tiny sizes, plus
closed forms: zero upstream gradients, alpha = 0 (phi drops out of the logits), n = 1
(H_res = 1 whatever the logit), t_max = 0 (H_res = exp(l_res)), linearity in the upstream
gradients, and the RMSNorm scale invariance of the projection."""
import numpy as np
import pytest

import oracle


def _problem(T, n, d, seed, alpha=0.7):
    rng = np.random.default_rng(seed)
    m = n * n + 2 * n
    return dict(
        X=rng.normal(size=(T, n, d)), F=rng.normal(size=(T, d)),
        phi=rng.normal(size=(n * d, m)) / np.sqrt(n * d),
        b_pre=rng.normal(size=n) * 0.3, b_post=rng.normal(size=n) * 0.3,
        b_res=np.eye(n) + rng.normal(size=(n, n)) * 0.3,
        alpha=np.array([alpha, 0.8 * alpha, 1.1 * alpha]),
        dY=rng.normal(size=(T, n, d)), dx=rng.normal(size=(T, d)))


def _loss(p, t_max):
    x_in, H = oracle.mhc_pre(p["X"], p["phi"], p["b_pre"], p["b_post"], p["b_res"],
                             *p["alpha"], eps=1e-20, t_max=t_max)
    Y = oracle.mhc_post(p["X"], p["F"], H)
    return float(np.sum(p["dY"] * Y) + np.sum(p["dx"] * x_in))


def _grads(p, t_max):
    return oracle.mhc_backward(p["X"], p["F"], p["phi"], p["b_pre"], p["b_post"], p["b_res"],
                               *p["alpha"], p["dY"], p["dx"], eps=1e-20, t_max=t_max)


# which gradient belongs to which input
_PAIRS = [("X", "dX"), ("F", "dF_out"), ("phi", "dphi"), ("b_pre", "db_pre"),
          ("b_post", "db_post"), ("b_res", "db_res"), ("alpha", "dalpha")]


@pytest.mark.parametrize("n,d,t_max", [(1, 4, 20), (2, 3, 20), (3, 5, 3), (4, 3, 20),
                                       (2, 4, 0), (3, 3, 1)])
def test_backward_matches_central_differences(n, d, t_max):
    p = _problem(2, n, d, seed=10 * n + d + t_max)
    g = _grads(p, t_max)
    step = 1e-6
    for name, gname in _PAIRS:
        a = p[name]
        fd = np.zeros(a.shape)
        for idx in np.ndindex(a.shape):
            keep = a[idx]
            a[idx] = keep + step
            lp = _loss(p, t_max)
            a[idx] = keep - step
            lm = _loss(p, t_max)
            a[idx] = keep
            fd[idx] = (lp - lm) / (2 * step)
        got = np.asarray(g[gname]).reshape(a.shape)
        err = np.abs(got - fd)
        assert (err <= 2e-7 * (1 + np.abs(fd))).all(), (name, err.max())


def test_zero_upstream_gives_zero_gradients():
    p = _problem(3, 4, 6, seed=1)
    p["dY"][:] = 0
    p["dx"][:] = 0
    for v in _grads(p, 20).values():
        assert np.all(v == 0)


def test_alpha_zero_removes_phi():
    """alpha = 0: the logits are the biases alone, so no gradient reaches phi, and the
    only path from X to the outputs is the read map and the merge (no RMSNorm term)."""
    p = _problem(3, 4, 5, seed=2, alpha=0.0)
    g = _grads(p, 20)
    assert np.all(g["dphi"] == 0)
    x_in, H = oracle.mhc_pre(p["X"], p["phi"], p["b_pre"], p["b_post"], p["b_res"], 0, 0, 0)
    Hp, Hr, Hq = oracle.split_H(H, 4)
    dX = np.einsum("tij,tic->tjc", Hr, p["dY"]) + Hp[:, :, None] * p["dx"][:, None, :]
    assert np.allclose(g["dX"], dX, rtol=0, atol=1e-13)
    assert np.allclose(g["dF_out"], np.einsum("ti,tic->tc", Hq, p["dY"]), rtol=0, atol=1e-13)


def test_n1_res_logit_has_no_gradient():
    """n = 1: H_res = exp(l)/exp(l) = 1 whatever l, so b_res and alpha_res get none."""
    p = _problem(4, 1, 6, seed=3)
    g = _grads(p, 20)
    assert np.all(np.abs(g["db_res"]) < 1e-15)
    assert abs(g["dalpha"][2]) < 1e-15


def test_tmax0_sinkhorn_is_exp():
    """t_max = 0: H_res = exp(l_res), so dL/dl_res = dH_res * H_res with
    dH_res[i][j] = sum_c dY[i,c] X[j,c]; with a single token db_res equals it."""
    p = _problem(1, 3, 4, seed=4)
    g = _grads(p, 0)
    _, H = oracle.mhc_pre(p["X"], p["phi"], p["b_pre"], p["b_post"], p["b_res"], *p["alpha"],
                          t_max=0)
    Hr = oracle.split_H(H, 3)[1][0]
    dHr = np.einsum("ic,jc->ij", p["dY"][0], p["X"][0])
    assert np.allclose(g["db_res"], dHr * Hr, rtol=1e-13, atol=1e-15)


def test_linear_in_upstream_gradients():
    p = _problem(3, 4, 5, seed=5)
    q = dict(p)
    rng = np.random.default_rng(9)
    q["dY"], q["dx"] = rng.normal(size=p["dY"].shape), rng.normal(size=p["dx"].shape)
    r = dict(p)
    r["dY"], r["dx"] = 2.0 * p["dY"] - 3.0 * q["dY"], 2.0 * p["dx"] - 3.0 * q["dx"]
    gp, gq, gr = _grads(p, 20), _grads(q, 20), _grads(r, 20)
    for k in gp:
        assert np.allclose(gr[k], 2.0 * gp[k] - 3.0 * gq[k], rtol=1e-10, atol=1e-12), k


def test_projection_is_scale_invariant_and_feeds_the_gates():
    """h(cX) = h(X) (RMSNorm, eps negligible), and H_pre = sigmoid(alpha_pre h_pre + b_pre)."""
    p = _problem(3, 4, 5, seed=6)
    h = oracle.mhc_projection(p["X"], p["phi"])
    assert np.allclose(oracle.mhc_projection(7.5 * p["X"], p["phi"]), h, rtol=1e-12, atol=1e-14)
    _, H = oracle.mhc_pre(p["X"], p["phi"], p["b_pre"], p["b_post"], p["b_res"], *p["alpha"])
    Hp = 1.0 / (1.0 + np.exp(-(p["alpha"][0] * h[:, :4] + p["b_pre"])))
    assert np.allclose(H[:, :4], Hp, rtol=1e-14, atol=1e-15)


def test_parameter_gradients_are_token_sums_independent_of_threads():
    """dphi, db and dalpha are sums over tokens: the oracle over all tokens equals, bit for
    bit, itself on 1, 3 and 8 threads, and agrees with the sum of per-token oracle calls."""
    p = _problem(37, 3, 5, seed=12)
    s = dict(eps=1e-20, t_max=20)

    def run(X, F, dY, dx, k):
        return oracle.mhc_backward(X, F, p["phi"], p["b_pre"], p["b_post"], p["b_res"], *p["alpha"],
                                   dY, dx, nthreads=k, **s)
    runs = [run(p["X"], p["F"], p["dY"], p["dx"], k) for k in (1, 3, 8)]
    for k in runs[0]:
        assert all(np.array_equal(runs[0][k], r[k]) for r in runs[1:]), k
    per_token = [run(p["X"][t:t + 1], p["F"][t:t + 1], p["dY"][t:t + 1], p["dx"][t:t + 1], 1) for t in range(37)]
    for k in ("dphi", "db_pre", "db_post", "db_res", "dalpha"):
        total = sum(g[k] for g in per_token)
        assert np.allclose(runs[0][k], total, rtol=1e-12, atol=1e-14 * np.abs(total).max()), k
