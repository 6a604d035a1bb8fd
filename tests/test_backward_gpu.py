"""GPU parity of the backward (mhc_pre_train + mhc_backward, through the C ABI) against the
fp64 oracle's reverse mode on the same seeded inputs.

Tolerances, from the arithmetic: every GPU step runs in fp32 on inputs that both sides read
exactly (bf16 inputs are exact in fp64), so a gradient entry differs from the oracle by a
few fp32 roundings of its terms, amplified at most tenfold by the 20 Sinkhorn rounds.  For
outputs stored in bf16 (dX, dF_out) the final rounding adds 2^-8 relative.  Each tensor is
checked entry by entry as |gpu - ref| <= rtol |ref| + atol * max|ref|:
  fp32 I/O     rtol 1e-4,            atol 1e-5
  bf16 I/O     dX, dF_out: rtol 2^-8 * 1.01, atol 2e-3; parameter gradients (fp32 sums over
               tokens of bf16-exact inputs): rtol 1e-3, atol 1e-4."""
import dataclasses

import numpy as np
import pytest

import oracle
from mhc_hyper_connections_b200 import workloads as wl

from _parity import torch_inputs

torch = pytest.importorskip("torch")
mhc = pytest.importorskip("mhc_hyper_connections_b200")

pytestmark = pytest.mark.gpu

GRADS = ("dX", "dF_out", "dphi", "db_pre", "db_post", "db_res", "dalpha")


def _upstream(w, seed):
    """dX_out, dx_in ~ N(0,1) in the workload's storage format (bf16 bits or fp32)."""
    rng = np.random.default_rng(seed)
    dY = rng.standard_normal((w.T, w.n, w.d), dtype=np.float32)
    dx = rng.standard_normal((w.T, w.d), dtype=np.float32)
    if w.dtype == "bf16":
        dY, dx = wl.bf16_round_bits(dY), wl.bf16_round_bits(dx)
    return dY, dx


def _dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_gpu(w, dY, dx, tokens=None, rows=None):
    """Training forward then backward on the GPU; returns a dict of float64 numpy
    gradients plus the saved projection h.  rows: the token rows of dX, dF_out and h to
    copy back (all by default; an empty array copies none)."""
    idx = np.arange(w.T) if tokens is None else np.asarray(tokens)
    sub = w.tokens(idx) if tokens is not None else w
    T, n, d, m = sub.T, sub.n, sub.d, sub.m
    t = torch_inputs(sub)
    X, F = t["X"], t["F"]
    s = sub.scalars()
    x_in = torch.empty(T, d, dtype=X.dtype, device="cuda")
    H = torch.empty(T, m, device="cuda")
    h = torch.empty(T, m, device="cuda")
    mhc.mhc_pre_train(X, t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"],
                      s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"], x_in, H, h)
    out = dict(dX=torch.empty_like(X), dF_out=torch.empty_like(F),
               dphi=torch.empty(n * d, m, device="cuda"), db_pre=torch.empty(n, device="cuda"),
               db_post=torch.empty(n, device="cuda"), db_res=torch.empty(n, n, device="cuda"),
               dalpha=torch.empty(3, device="cuda"))
    ws = torch.empty(max(1, mhc.mhc_backward_workspace_bytes(T, n, d)), dtype=torch.uint8, device="cuda")
    mhc.mhc_backward(X, F, t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"],
                     s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"], H, h, _dev(dY[idx]),
                     _dev(dx[idx]), out["dX"], out["dF_out"], out["dphi"], out["db_pre"],
                     out["db_post"], out["db_res"], out["dalpha"], ws)
    torch.cuda.synchronize()
    out["h"] = h
    sel = None if rows is None else torch.from_numpy(np.asarray(rows, dtype=np.int64)).cuda()
    res = {}
    for k, v in out.items():
        if sel is not None and k in ("dX", "dF_out", "h"):
            v = v[sel]
        res[k] = v.double().cpu().numpy()
    return res


def run_oracle(w, dY, dx, tokens=None, nthreads=8):
    idx = np.arange(w.T) if tokens is None else np.asarray(tokens)
    sub = w.tokens(idx) if tokens is not None else w
    s = sub.scalars()
    return oracle.mhc_backward(sub.values(sub.X), sub.values(sub.F_out), sub.phi, sub.b_pre,
                               sub.b_post, sub.b_res, s["alpha_pre"], s["alpha_post"],
                               s["alpha_res"], w.values(dY[idx]), w.values(dx[idx]),
                               eps=s["eps"], t_max=s["t_max"], nthreads=nthreads)


def _tols(dtype, name):
    if dtype == "f32":
        return 1e-4, 1e-5
    if name in ("dX", "dF_out"):
        return 2.0 ** -8 * 1.01, 2e-3
    return 1e-3, 1e-4


def check(w, gpu, ref, what, names=GRADS):
    for k in names:
        g, r = np.asarray(gpu[k]).reshape(-1), np.asarray(ref[k]).reshape(-1)
        rtol, atol = _tols(w.dtype, k)
        scale = max(np.abs(r).max(), 1e-30)
        bad = np.abs(g - r) > rtol * np.abs(r) + atol * scale
        assert not bad.any(), (what, k, int(bad.sum()), float(np.abs(g - r).max() / scale))


def test_tiny_f32_full():
    w = wl.make_config("tiny_f32_T64_n4_d64")
    dY, dx = _upstream(w, 100)
    check(w, run_gpu(w, dY, dx), run_oracle(w, dY, dx), "tiny")


def test_bf16_d1024_full():
    w = wl.make_config("bf16_T4096_n4_d1024")
    dY, dx = _upstream(w, 101)
    check(w, run_gpu(w, dY, dx), run_oracle(w, dY, dx, nthreads=16), "d1024")


@pytest.mark.parametrize("T,n,d,dt", [(1, 1, 8, "bf16"), (33, 2, 24, "f32"), (100, 3, 136, "bf16"),
                                      (37, 4, 64, "bf16"), (300, 1, 1024, "bf16"), (65, 3, 12, "f32"),
                                      (129, 3, 192, "bf16"), (1000, 2, 640, "bf16"), (64, 4, 128, "bf16"),
                                      (200, 4, 4096, "bf16"), (1, 2, 64, "bf16"), (777, 1, 128, "bf16"),
                                      (64, 4, 12800, "bf16"), (100, 2, 9600, "bf16"), (50, 1, 25600, "bf16")])
def test_shapes(T, n, d, dt):
    """Ragged shapes on both dX / dphi kernels: bf16 with d a multiple of 64 takes the
    tensor-core step (token tails inside a stage, groups that end mid-tensor or hold no
    tokens, odd n with a placeholder stream, and wide d: 150 to 400 channel slices), the rest
    the CUDA-core step."""
    w = wl.make_inputs(T=T, n=n, d=d, dtype=dt, seed=T * 7 + n * 3 + d, alpha=0.3)
    dY, dx = _upstream(w, T + d)
    check(w, run_gpu(w, dY, dx), run_oracle(w, dY, dx), f"T{T} n{n} d{d} {dt}")


@pytest.mark.parametrize("t_max,n", [(0, 4), (1, 4), (3, 3), (21, 4), (41, 2), (64, 4)])
def test_sinkhorn_depths(t_max, n):
    """Sinkhorn depths other than 20: none (H_res = exp of the logits), one round, and depths
    past the 20 round inputs the backward keeps per token, where it keeps every 2nd, 3rd or
    4th and replays the rounds in between."""
    w = wl.make_inputs(T=70, n=n, d=40, dtype="bf16", seed=500 + t_max, alpha=0.3)
    w = dataclasses.replace(w, t_max=t_max)
    dY, dx = _upstream(w, 600 + t_max)
    check(w, run_gpu(w, dY, dx), run_oracle(w, dY, dx), f"t_max {t_max} n {n}")


@pytest.mark.parametrize("t_max", [0, 1, 41])
def test_sinkhorn_depths_tensor_core_step(t_max):
    """The same depths with d a multiple of 64, so the tensor-core dX / dphi step runs."""
    w = wl.make_inputs(T=150, n=4, d=128, dtype="bf16", seed=700 + t_max, alpha=0.3)
    w = dataclasses.replace(w, t_max=t_max)
    dY, dx = _upstream(w, 800 + t_max)
    check(w, run_gpu(w, dY, dx), run_oracle(w, dY, dx), f"t_max {t_max} tensor-core step")


def test_headline_size_sampled_and_additive():
    """Backward at the forward-plus-backward workload (T=16384, n=4, d=4096, bf16 with outlier
    channels): dX and dF_out on sampled tokens against the oracle on those tokens (they depend
    only on their own token); the parameter gradients on a 512-token subset against the
    oracle; and, at full size, additivity of the parameter gradients over the two token
    halves."""
    w = wl.make_config(wl.HEADLINE)
    dY, dx = _upstream(w, 102)
    rng = np.random.default_rng(7)
    idx = np.unique(np.concatenate([np.arange(4), np.arange(w.T - 4, w.T), rng.choice(w.T, 24, replace=False)]))
    full = run_gpu(w, dY, dx, rows=idx)
    ref = run_oracle(w, dY, dx, tokens=idx, nthreads=16)
    check(w.tokens(idx), full, ref, "headline sampled", names=("dX", "dF_out"))
    part = np.arange(512) * 31 % w.T
    part = np.unique(part)
    check(w.tokens(part), run_gpu(w, dY, dx, tokens=part, rows=[]), run_oracle(w, dY, dx, tokens=part, nthreads=16),
          "headline 512-token subset", names=("dphi", "db_pre", "db_post", "db_res", "dalpha"))
    half = w.T // 2
    a = run_gpu(w, dY, dx, tokens=np.arange(half), rows=[])
    b = run_gpu(w, dY, dx, tokens=np.arange(half, w.T), rows=[])
    for k in ("dphi", "db_pre", "db_post", "db_res", "dalpha"):
        scale = np.abs(full[k]).max()
        assert np.abs(a[k] + b[k] - full[k]).max() <= 1e-4 * scale, k
    assert all(np.isfinite(full[k]).all() for k in GRADS)


def test_headline_size_all_tokens():
    """The forward-plus-backward workload at full size (T=16384, n=4, d=4096, bf16 with
    outlier channels): the parameter gradients, summed on the GPU over all 16384 tokens,
    against the oracle's sums over all tokens (run in token chunks, the chunk sums added in
    token order); dX and dF_out on 1056 tokens (the first 16, the last 16 and 1024 drawn)."""
    import os
    w = wl.make_config(wl.HEADLINE)
    dY, dx = _upstream(w, 105)
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([np.arange(16), np.arange(w.T - 16, w.T),
                                     rng.choice(np.arange(16, w.T - 16), 1024, replace=False)]))
    full = run_gpu(w, dY, dx, rows=rows)
    cores = os.cpu_count() or 8
    params = ("dphi", "db_pre", "db_post", "db_res", "dalpha")
    ref = {k: 0.0 for k in params}
    for c0 in range(0, w.T, 2048):
        part = run_oracle(w, dY, dx, tokens=np.arange(c0, min(w.T, c0 + 2048)), nthreads=cores)
        for k in params:
            ref[k] = ref[k] + part[k]
    check(w, full, ref, "headline all tokens", names=params)
    check(w.tokens(rows), full, run_oracle(w, dY, dx, tokens=rows, nthreads=cores),
          "headline 1056 tokens", names=("dX", "dF_out"))


def test_saved_projection_matches_oracle_on_both_paths():
    for name in ("tiny_f32_T64_n4_d64", "bf16_T4096_n4_d1024"):
        w = wl.make_config(name)
        dY, dx = _upstream(w, 103)
        h = run_gpu(w, dY, dx)["h"]
        ref = oracle.mhc_projection(w.values(w.X), w.phi, eps=w.scalars()["eps"])
        scale = np.abs(ref).max()
        tol = 1e-5 if w.dtype == "f32" else 2e-3
        assert np.abs(h - ref).max() <= tol * scale, name


def test_train_forward_equals_forward():
    """mhc_pre_train writes the same x_in and H as mhc_pre (bitwise), on the path mhc_pre takes."""
    w = wl.make_inputs(T=300, n=4, d=2048, dtype="bf16", seed=5)
    t = torch_inputs(w)
    X, phi, bp, bq, br = t["X"], t["phi"], t["b_pre"], t["b_post"], t["b_res"]
    s = w.scalars()
    outs = []
    for train in (False, True):
        x_in = torch.empty(w.T, w.d, dtype=torch.bfloat16, device="cuda")
        H = torch.empty(w.T, w.m, device="cuda")
        args = (X, phi, bp, bq, br, s["alpha_pre"], s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"], x_in, H)
        if train:
            mhc.mhc_pre_train(*args, torch.empty(w.T, w.m, device="cuda"))
        else:
            mhc.mhc_pre(*args)
        outs.append((x_in, H))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_deterministic_bitwise():
    w = wl.make_inputs(T=700, n=4, d=512, dtype="bf16", seed=11, alpha=0.2)
    dY, dx = _upstream(w, 104)
    a, b = run_gpu(w, dY, dx), run_gpu(w, dY, dx)
    for k in GRADS:
        assert np.array_equal(a[k], b[k]), k


def test_errors_and_empty():
    w = wl.make_inputs(T=8, n=4, d=64, dtype="bf16", seed=2)
    X = _dev(w.X)
    z = lambda *s: torch.zeros(*s, device="cuda")
    f = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device="cuda")
    m = w.m
    base = dict(X=X, F_out=f(8, 64), phi=z(256, m), b_pre=z(4), b_post=z(4), b_res=z(4, 4),
                alpha_pre=0.1, alpha_post=0.1, alpha_res=0.1, eps=1e-20, t_max=20, H=z(8, m), h=z(8, m),
                dX_out=f(8, 4, 64), dx_in=f(8, 64), dX=f(8, 4, 64), dF_out=f(8, 64), dphi=z(256, m),
                db_pre=z(4), db_post=z(4), db_res=z(4, 4), dalpha=z(3))
    need = mhc.mhc_backward_workspace_bytes(8, 4, 64)
    with pytest.raises(mhc.MhcError, match="WORKSPACE"):
        mhc.mhc_backward(**base, workspace=torch.empty(need - 256, dtype=torch.uint8, device="cuda"))
    assert mhc.mhc_backward_workspace_bytes(8, 5, 64) == 0
    # T = 0: the parameter gradients become zero
    e = dict(base)
    for k in ("dphi", "db_pre", "db_post", "db_res", "dalpha"):
        e[k] = torch.full_like(base[k], 7.0)
    for k in ("X", "dX_out", "dX"):
        e[k] = f(0, 4, 64)
    for k in ("F_out", "dx_in", "dF_out"):
        e[k] = f(0, 64)
    e["H"], e["h"] = z(0, m), z(0, m)
    mhc.mhc_backward(**e, workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    for k in ("dphi", "db_pre", "db_post", "db_res", "dalpha"):
        assert (e[k] == 0).all(), k
