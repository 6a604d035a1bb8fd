"""The binding's shape checks, on the CPU: mhc_backward and mhc_backward_noalloc, and the
forward bindings mhc_pre, mhc_pre_train and mhc_post.

The C ABI receives only pointers, so the binding checks every tensor's shape before a
call: a tensor smaller than the backward expects would be read or written past its end.
The tensors here are CPU tensors.  A call whose shapes pass gets as far as the device
check, which refuses it ("must be a CUDA tensor"); a call with a wrong shape is refused
earlier, naming the tensor.  The accepted cases build their tensors the way the GPU tests,
the benchmark and the smoke test do."""
import dataclasses

import pytest

from mhc_hyper_connections_b200 import workloads as wl

from _parity import torch_inputs

torch = pytest.importorskip("torch")
mhc = pytest.importorskip("mhc_hyper_connections_b200")

SCALARS = (0.1, 0.1, 0.1, 1e-20, 20)


def _args(w):
    """(X, F_out, phi, b_pre, b_post, b_res, H, h, dX_out, dx_in, dX, dF_out, dphi, db_pre,
    db_post, db_res, dalpha) as the GPU backward tests build them, on the CPU."""
    t = torch_inputs(w, device="cpu")
    T, n, d, m = w.T, w.n, w.d, w.m
    X, F = t["X"], t["F"]
    return dict(X=X, F_out=F, phi=t["phi"], b_pre=t["b_pre"], b_post=t["b_post"], b_res=t["b_res"],
                H=torch.empty(T, m), h=torch.empty(T, m), dX_out=torch.empty_like(X),
                dx_in=torch.empty_like(F), dX=torch.empty_like(X), dF_out=torch.empty_like(F),
                dphi=torch.empty(n * d, m), db_pre=torch.empty(n), db_post=torch.empty(n),
                db_res=torch.empty(n, n), dalpha=torch.empty(3))


def _call(a, noalloc=False):
    pos = (a["X"], a["F_out"], a["phi"], a["b_pre"], a["b_post"], a["b_res"], *SCALARS, a["H"], a["h"],
           a["dX_out"], a["dx_in"], a["dX"], a["dF_out"], a["dphi"], a["db_pre"], a["db_post"],
           a["db_res"], a["dalpha"])
    if noalloc:
        mhc.mhc_backward_noalloc(*pos)
    else:
        mhc.mhc_backward(*pos, torch.empty(256, dtype=torch.uint8))


CASES = [wl.make_config("tiny_f32_T64_n4_d64"),
         wl.make_inputs(T=1, n=1, d=8, dtype="bf16", seed=1),
         wl.make_inputs(T=33, n=2, d=24, dtype="f32", seed=2),
         wl.make_inputs(T=100, n=3, d=136, dtype="bf16", seed=3),
         dataclasses.replace(wl.make_inputs(T=70, n=2, d=40, dtype="bf16", seed=4), t_max=41),
         wl.make_inputs(T=0, n=4, d=64, dtype="bf16", seed=5)]


@pytest.mark.parametrize("noalloc", [False, True])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_shapes_of_the_gpu_tests_pass_the_check(w, noalloc):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        _call(_args(w), noalloc)


def test_bench_and_no_alloc_test_shapes_pass_the_check():
    # bench.py's backward step: bf16 X [T, n, d], upstream dX_out [T, n, d] and dx_in [T, d]
    w = wl.make_inputs(T=48, n=4, d=128, dtype="bf16", seed=6)
    a = _args(w)
    a["dX_out"] = torch.empty(w.T, w.n, w.d, dtype=torch.bfloat16)
    a["dx_in"] = torch.empty(w.T, w.d, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        _call(a)
    # the no-alloc test's oversize case: n = 1, d = 8, zero-filled fp32 parameters
    T, n, d, m = 1000, 1, 8, 3
    X = torch.zeros(T, n, d, dtype=torch.bfloat16)
    F = torch.zeros(T, d, dtype=torch.bfloat16)
    z = lambda *sh: torch.zeros(*sh)
    b = dict(X=X, F_out=F, phi=z(n * d, m), b_pre=z(n), b_post=z(n), b_res=z(n, n), H=z(T, m), h=z(T, m),
             dX_out=torch.zeros_like(X), dx_in=torch.zeros_like(F), dX=torch.zeros_like(X),
             dF_out=torch.zeros_like(F), dphi=z(n * d, m), db_pre=z(n), db_post=z(n), db_res=z(n, n),
             dalpha=z(3))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        _call(b, noalloc=True)


@pytest.mark.parametrize("noalloc", [False, True])
@pytest.mark.parametrize("name,bad", [
    ("dphi", lambda w: torch.empty(w.n * w.d - 1, w.m)),
    ("phi", lambda w: torch.empty(w.m, w.n * w.d)),
    ("dX", lambda w: torch.empty(w.T, w.n, w.d - 8, dtype=torch.bfloat16)),
    ("dX_out", lambda w: torch.empty(w.T - 1, w.n, w.d, dtype=torch.bfloat16)),
    ("F_out", lambda w: torch.empty(w.T, w.n * w.d, dtype=torch.bfloat16)),
    ("dx_in", lambda w: torch.empty(w.T * w.d, dtype=torch.bfloat16)),
    ("dF_out", lambda w: torch.empty(w.T, 1, w.d, dtype=torch.bfloat16)),
    ("H", lambda w: torch.empty(w.T, w.m - 1)),
    ("h", lambda w: torch.empty(w.T + 1, w.m)),
    ("db_res", lambda w: torch.empty(w.n)),
    ("b_res", lambda w: torch.empty(w.n, w.n + 1)),
    ("db_pre", lambda w: torch.empty(w.n + 1)),
    ("b_post", lambda w: torch.empty(1)),
    ("dalpha", lambda w: torch.empty(2)),
])
def test_wrong_shapes_are_refused_by_name(name, bad, noalloc):
    w = wl.make_inputs(T=16, n=4, d=64, dtype="bf16", seed=7)
    a = _args(w)
    a[name] = bad(w)
    with pytest.raises(ValueError, match=rf"{name} (has shape|needs)"):
        _call(a, noalloc)


def test_flat_bias_vectors_are_accepted():
    # b_res and db_res are read as n*n values: [n, n] and [n*n] both hold them
    w = wl.make_inputs(T=16, n=3, d=32, dtype="bf16", seed=8)
    a = _args(w)
    a["b_res"] = a["b_res"].reshape(-1)
    a["db_res"] = torch.empty(w.n * w.n)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        _call(a)


def test_X_must_be_three_dimensional():
    w = wl.make_inputs(T=16, n=4, d=64, dtype="bf16", seed=9)
    a = _args(w)
    a["X"] = a["X"].reshape(w.T, -1)
    with pytest.raises(ValueError, match=r"X must be \[T, n, d\]"):
        _call(a)


def _fwd(w):
    t = torch_inputs(w, device="cpu")
    return (t, torch.empty(w.T, w.d, dtype=t["X"].dtype), torch.empty(w.T, w.m), torch.empty(w.T, w.m),
            torch.empty_like(t["X"]))


@pytest.mark.parametrize("w", CASES[:4] + [wl.make_inputs(T=9, n=8, d=16, dtype="bf16", seed=10)],
                         ids=lambda w: w.name)
def test_forward_shapes_of_the_gpu_tests_pass_the_check(w):
    t, x_in, H, h, Y = _fwd(w)
    sc = (0.01, 0.01, 0.01, 1e-20, 20)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        mhc.mhc_pre(t["X"], t["phi"], t["b_pre"], t["b_post"], t["b_res"], *sc, x_in, H)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        mhc.mhc_pre_train(t["X"], t["phi"], t["b_pre"], t["b_post"], t["b_res"], *sc, x_in, H, h)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        mhc.mhc_post(t["X"], t["F"], H, Y)


@pytest.mark.parametrize("fn", ["mhc_pre", "mhc_pre_train"])
@pytest.mark.parametrize("name,bad,msg", [
    ("phi", lambda w: torch.empty(w.n * w.d, w.m + 1), "shapes must be"),
    ("x_in", lambda w: torch.empty(w.T, w.d - 1, dtype=torch.bfloat16), "shapes must be"),
    ("H", lambda w: torch.empty(w.T - 1, w.m), "shapes must be"),
    ("b_pre", lambda w: torch.empty(w.n - 1), "need n entries"),
    ("b_post", lambda w: torch.empty(w.n + 1), "need n entries"),
    ("b_res", lambda w: torch.empty(w.n), "need n entries"),
])
def test_forward_wrong_shapes_are_refused(fn, name, bad, msg):
    w = wl.make_inputs(T=16, n=4, d=64, dtype="bf16", seed=11)
    t, x_in, H, h, _ = _fwd(w)
    a = dict(X=t["X"], phi=t["phi"], b_pre=t["b_pre"], b_post=t["b_post"], b_res=t["b_res"], x_in=x_in, H=H)
    a[name] = bad(w)
    extra = (h,) if fn == "mhc_pre_train" else ()
    with pytest.raises(ValueError, match=f"{fn}: .*{msg}"):
        getattr(mhc, fn)(a["X"], a["phi"], a["b_pre"], a["b_post"], a["b_res"], 0.01, 0.01, 0.01, 1e-20, 20,
                         a["x_in"], a["H"], *extra)


def test_pre_train_checks_h():
    w = wl.make_inputs(T=16, n=4, d=64, dtype="bf16", seed=12)
    t, x_in, H, _, _ = _fwd(w)
    with pytest.raises(ValueError, match="mhc_pre_train: shapes must be"):
        mhc.mhc_pre_train(t["X"], t["phi"], t["b_pre"], t["b_post"], t["b_res"], 0.01, 0.01, 0.01, 1e-20, 20,
                          x_in, H, torch.empty(w.T, w.m - 1))


@pytest.mark.parametrize("name", ["F_out", "H", "X_out"])
def test_post_wrong_shapes_are_refused(name):
    w = wl.make_inputs(T=16, n=4, d=64, dtype="bf16", seed=13)
    t, _, H, _, Y = _fwd(w)
    a = dict(F_out=t["F"], H=H, X_out=Y)
    a[name] = {"F_out": torch.empty(w.T, w.d + 8, dtype=torch.bfloat16), "H": torch.empty(w.T, w.m - 2),
               "X_out": torch.empty(w.T, w.n - 1, w.d, dtype=torch.bfloat16)}[name]
    with pytest.raises(ValueError, match="mhc_post: shapes must be"):
        mhc.mhc_post(t["X"], a["F_out"], a["H"], a["X_out"])
