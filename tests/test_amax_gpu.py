"""GPU parity of mhc_amax_gain (the Amax Gain Magnitude of composite residual maps) against
the oracle, on stacks of raw near-identity maps (the HC-like case whose gain grows with
depth, as in the slavadubrov.com demo), on Sinkhorn-projected maps, and on coefficient rows
that mhc_pre itself wrote for consecutive layers.  The GPU multiplies in fp32: a product of
L maps carries about L fp32 roundings, so gains are compared with relative tolerance 2e-4."""
import numpy as np
import pytest

import oracle
from mhc_hyper_connections_b200 import workloads as wl

from _parity import torch_inputs

torch = pytest.importorskip("torch")
mhc = pytest.importorskip("mhc_hyper_connections_b200")

pytestmark = pytest.mark.gpu


def _gpu_gain(Hs):
    H = torch.from_numpy(np.ascontiguousarray(Hs, dtype=np.float32)).cuda()
    g = torch.empty(Hs.shape[0], Hs.shape[1], 2, device="cuda")
    mhc.mhc_amax_gain(H, g)
    torch.cuda.synchronize()
    return g.double().cpu().numpy()


def _check(Hs):
    Hs32 = Hs.astype(np.float32)
    ref = oracle.amax_gain(Hs32.astype(np.float64))
    got = _gpu_gain(Hs32)
    assert (np.abs(got - ref) <= 2e-4 * np.abs(ref)).all(), np.abs(got / ref - 1).max()
    return ref


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_raw_and_sinkhorn_stacks(n):
    rng = np.random.default_rng(n)
    L, T, m = 60, 3001, n * n + 2 * n
    Hs = rng.normal(size=(L, T, m))
    A = np.eye(n) + 0.3 * rng.standard_normal((L, T, n, n))
    Hs[:, :, n:n + n * n] = A.reshape(L, T, n * n)
    raw = _check(Hs)
    if n > 1:
        assert raw[-1].max() > 10.0                   # the raw product grows with depth
    S = np.array([[oracle.sinkhorn(A[l, t], 20) for t in range(0, T, 500)] for l in range(L)])
    Hk = Hs[:, ::500].copy()
    Hk[:, :, n:n + n * n] = S.reshape(L, -1, n * n)
    sk = _check(Hk)
    assert sk.max() < 1.1                             # nearly doubly stochastic: gain near 1


def test_layers_written_by_mhc_pre():
    """Eight layers' H from mhc_pre on independent inputs (n = 4, d = 1024)."""
    layers = []
    for l in range(8):
        w = wl.make_inputs(T=1000, n=4, d=1024, dtype="bf16", seed=50 + l, alpha=0.5)
        t = torch_inputs(w)
        s = w.scalars()
        x_in = torch.empty(w.T, w.d, dtype=torch.bfloat16, device="cuda")
        H = torch.empty(w.T, w.m, device="cuda")
        mhc.mhc_pre(t["X"], t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"],
                    s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"], x_in, H)
        layers.append(H)
    Hs = torch.stack(layers).contiguous()
    g = torch.empty(8, 1000, 2, device="cuda")
    mhc.mhc_amax_gain(Hs, g)
    torch.cuda.synchronize()
    ref = oracle.amax_gain(Hs.double().cpu().numpy())
    got = g.double().cpu().numpy()
    assert (np.abs(got - ref) <= 2e-4 * np.abs(ref)).all()
    assert got[:, :, 0].max() < 1.0 + 1e-4            # rows sum to 1 after the last row step
