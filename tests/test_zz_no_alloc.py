"""mhc_backward_noalloc, the backward for callers that cannot allocate device memory (a
plugin handed device pointers by a framework that owns all allocations through its own
pool, or a call site where a device-synchronising cudaMalloc is not allowed).  It works in
a fixed scratch array inside the library instead of a caller workspace.

Checked through the C ABI against mhc_backward with a caller workspace on two calls in a
row.  Both run the same deterministic kernels, so every output must be bitwise equal.  The
larger problem runs first and the smaller second, so the second call finds the first
call's stale contents in the part of the array it uses.  Sizes beyond the array are
refused.  This file is collected last, and passes alone in a fresh process as well as
after the other tests."""
import numpy as np
import pytest

from mhc_hyper_connections_b200 import workloads as wl

from _parity import torch_inputs

torch = pytest.importorskip("torch")
mhc = pytest.importorskip("mhc_hyper_connections_b200")

pytestmark = pytest.mark.gpu

PARAMS = ("dphi", "db_pre", "db_post", "db_res", "dalpha")


def _upstream(w, seed):
    rng = np.random.default_rng(seed)
    dY = torch.from_numpy(rng.standard_normal((w.T, w.n, w.d), dtype=np.float32)).cuda()
    dx = torch.from_numpy(rng.standard_normal((w.T, w.d), dtype=np.float32)).cuda()
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return dY.to(dt), dx.to(dt)


def _problem(w, seed):
    t = torch_inputs(w)
    s = w.scalars()
    x_in = torch.empty(w.T, w.d, dtype=t["X"].dtype, device="cuda")
    H = torch.empty(w.T, w.m, device="cuda")
    h = torch.empty(w.T, w.m, device="cuda")
    mhc.mhc_pre_train(t["X"], t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"],
                      s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"], x_in, H, h)
    dY, dx = _upstream(w, seed)
    return t, s, H, h, dY, dx


def _grads(w, prob, noalloc):
    t, s, H, h, dY, dx = prob
    n, d, m = w.n, w.d, w.m
    out = dict(dX=torch.empty_like(t["X"]), dF_out=torch.empty_like(t["F"]),
               dphi=torch.empty(n * d, m, device="cuda"), db_pre=torch.empty(n, device="cuda"),
               db_post=torch.empty(n, device="cuda"), db_res=torch.empty(n, n, device="cuda"),
               dalpha=torch.empty(3, device="cuda"))
    args = (t["X"], t["F"], t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"],
            s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"], H, h, dY, dx, out["dX"],
            out["dF_out"], out["dphi"], out["db_pre"], out["db_post"], out["db_res"], out["dalpha"])
    if noalloc:
        mhc.mhc_backward_noalloc(*args)
    else:
        ws = torch.empty(mhc.mhc_backward_workspace_bytes(w.T, n, d), dtype=torch.uint8, device="cuda")
        mhc.mhc_backward(*args, ws)
    torch.cuda.synchronize()
    return {k: v.double().cpu().numpy() for k, v in out.items()}


def _equal(got, ref):
    """Same kernels, same inputs: bitwise equal outputs (NaN nowhere)."""
    for k, r in ref.items():
        assert np.isfinite(r).all(), k
        assert np.array_equal(got[k], r), k


def test_noalloc_matches_backward_on_two_calls_in_a_row():
    cases = [wl.make_inputs(T=4096, n=4, d=4096, dtype="bf16", seed=22, alpha=0.3, outlier_frac=0.01),
             wl.make_inputs(T=2048, n=4, d=1024, dtype="bf16", seed=21, alpha=0.2)]
    for i, w in enumerate(cases):
        assert mhc.mhc_backward_workspace_bytes(w.T, w.n, w.d) <= mhc.NOALLOC_SCRATCH_BYTES
        prob = _problem(w, 300 + i)
        _equal(_grads(w, prob, noalloc=True), _grads(w, prob, noalloc=False))


def test_noalloc_refuses_sizes_beyond_its_scratch():
    T, n, d = 1_000_000, 1, 8
    assert mhc.mhc_backward_workspace_bytes(T, n, d) > mhc.NOALLOC_SCRATCH_BYTES
    X = torch.zeros(T, n, d, dtype=torch.bfloat16, device="cuda")
    F = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    z = lambda *sh: torch.zeros(*sh, device="cuda")
    m = n * n + 2 * n
    with pytest.raises(mhc.MhcError, match="WORKSPACE"):
        mhc.mhc_backward_noalloc(X, F, z(n * d, m), z(n), z(n), z(n, n), 0.1, 0.1, 0.1, 1e-20, 20,
                                 z(T, m), z(T, m), torch.zeros_like(X), torch.zeros_like(F),
                                 torch.zeros_like(X), torch.zeros_like(F), z(n * d, m), z(n), z(n),
                                 z(n, n), z(3))
