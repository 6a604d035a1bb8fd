"""GPU parity of the HC comparison maps (mhc_pre_hc, then mhc_post) against the oracle's HC
pre stage and post merge, on every pre path the device runs; and the depth comparison the
pages draw between HC and mHC, measured with mhc_amax_gain on maps the GPU produced.

Tolerances are those of the mHC parity tests (tests/_parity.py): the HC maps run the same
fp32 projection, then b + alpha tanh instead of the gates and Sinkhorn."""
import numpy as np
import pytest

import oracle
from mhc_hyper_connections_b200 import workloads as wl

from _parity import check_against_oracle, to_f64, torch_inputs

torch = pytest.importorskip("torch")
mhc = pytest.importorskip("mhc_hyper_connections_b200")

pytestmark = pytest.mark.gpu


def _paths(w):
    dt = 1 if w.dtype == "bf16" else 0
    return [p for p in (mhc.PRE_GENERIC, mhc.PRE_CLUSTER_TC, mhc.PRE_TWO_PASS_TC)
            if mhc.mhc_pre_path_ok(w.T, w.n, w.d, dt, p)]


def run_gpu_hc(w, path, inputs=None):
    t = inputs if inputs is not None else torch_inputs(w)
    X = t["X"]
    x_in = torch.empty(w.T, w.d, dtype=X.dtype, device="cuda")
    H = torch.empty(w.T, w.m, device="cuda")
    Y = torch.empty_like(X)
    s = w.scalars()
    mhc.mhc_pre_hc(X, t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"],
                   s["alpha_post"], s["alpha_res"], s["eps"], x_in, H, path=path)
    mhc.mhc_post(X, t["F"], H, Y)
    torch.cuda.synchronize()
    assert mhc.mhc_device_status() == 0
    return x_in, H, Y


def run_oracle_hc(w):
    X, F = w.values(w.X), w.values(w.F_out)
    s = w.scalars()
    x_in, H = oracle.hc_pre(X, w.phi, w.b_pre, w.b_post, w.b_res, s["alpha_pre"], s["alpha_post"],
                            s["alpha_res"], eps=s["eps"], nthreads=8)
    return x_in, H, oracle.mhc_post(X, F, H, nthreads=8)


def _hc_inputs(T, n, d, dtype, seed, alpha):
    """HC's static maps start near the plain residual: b_res = I + noise, b_pre = 1/n,
    b_post = 1; the workload generator's b_res (4 I + noise) is mHC's logit bias."""
    w = wl.make_inputs(T=T, n=n, d=d, dtype=dtype, seed=seed, alpha=alpha)
    rng = np.random.default_rng(seed + 1)
    w.b_res = (np.eye(n) + 0.1 * rng.standard_normal((n, n))).astype(np.float32)
    w.b_pre = np.full(n, 1.0 / n, np.float32)
    w.b_post = np.ones(n, np.float32)
    return w


@pytest.mark.parametrize("T,n,d,dt,alpha", [
    (64, 4, 64, "f32", 0.3), (4096, 4, 1024, "bf16", 0.01), (130, 4, 4096, "bf16", 0.5),
    (77, 4, 2560, "bf16", 1.0), (33, 1, 1024, "bf16", 0.7), (50, 3, 1280, "bf16", 0.4),
    (19, 8, 64, "bf16", 0.5), (9, 2, 24, "f32", 0.9), (2000, 8, 4096, "bf16", 0.5),
    (400, 4, 8192, "bf16", 0.8),
])
def test_hc_maps_match_the_oracle(T, n, d, dt, alpha):
    w = _hc_inputs(T, n, d, dt, seed=T + 10 * n + d, alpha=alpha)
    ref = run_oracle_hc(w)
    t = torch_inputs(w)
    for p in _paths(w):
        check_against_oracle(w, run_gpu_hc(w, p, t), ref, f"HC T{T} n{n} d{d} {dt} path{p}")


def test_hc_has_signed_entries_and_no_doubly_stochastic_constraint():
    w = _hc_inputs(256, 4, 1024, "bf16", seed=3, alpha=1.0)
    for p in _paths(w):
        _, H, _ = run_gpu_hc(w, p)
        Hr = H[:, 4:20].reshape(-1, 4, 4)
        assert (Hr < 0).any()
        assert (Hr.sum(dim=2) - 1).abs().max().item() > 1e-2


def test_depth_gain_hc_grows_mhc_stays_bounded():
    """60 layers of maps from the GPU for the same tokens: the composite of HC residual maps
    grows with depth while mHC's stays near 1 (the comparison of the "DeepSeek-V4/mhc"
    page's stability paragraph and the slavadubrov.com numpy demo); the diagnostic kernel
    agrees with the oracle on these stacks."""
    L, T, n, d = 60, 256, 4, 1024
    hc, mh = [], []
    for layer in range(L):
        w = _hc_inputs(T, n, d, "bf16", seed=1000 + layer, alpha=0.3)
        rng = np.random.default_rng(layer)
        w.b_res = (np.eye(n) + 0.3 * rng.standard_normal((n, n))).astype(np.float32)
        _, H, _ = run_gpu_hc(w, mhc.PRE_AUTO)
        hc.append(H)
        m = wl.make_inputs(T=T, n=n, d=d, dtype="bf16", seed=1000 + layer)
        t = torch_inputs(m)
        s = m.scalars()
        x_in = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        Hm = torch.empty(T, m.m, device="cuda")
        mhc.mhc_pre(t["X"], t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"],
                    s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"], x_in, Hm)
        mh.append(Hm)
    gains = {}
    for name, stack in (("hc", torch.stack(hc)), ("mhc", torch.stack(mh))):
        g = torch.empty(L, T, 2, device="cuda")
        mhc.mhc_amax_gain(stack, g)
        torch.cuda.synchronize()
        gn = to_f64(g)
        ref = oracle.amax_gain(to_f64(stack))
        assert np.allclose(gn, ref, rtol=2e-3, atol=0), name
        gains[name] = gn[-1].max()
    assert gains["hc"] > 10.0, gains
    assert gains["mhc"] < 2.0, gains
