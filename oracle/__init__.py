"""fp64 CPU oracle for the mHC pre and post stages (ctypes wrapper around mhc_oracle.c).

TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the benchmark's
CPU-baseline / reference leg may import this module; the product path never does and
has no CPU fallback.  It shares no code with the CUDA library.

What each function follows (page title, section / equation):
  * sinkhorn  -- "DeepSeek-V4/mhc" page, equations sinkhorn-init and sinkhorn;
                 slavadubrov.com mHC article, section "Sinkhorn-Knopp-projectie".
  * mhc_pre   -- "DeepSeek-V4/mhc" page, "动态参数化怎么实现": equations rmsnorm,
                 a/b/c-tilde and gate; slavadubrov.com article Eq. 3 (read map).
  * hc_pre    -- the HC maps mHC is compared with: slavadubrov.com article,
                 "Kernmechanismen" (a bias plus an input-dependent term through tanh)
                 and "Details van de parameterisatie" (tanh is what mHC replaces).
  * mhc_post  -- slavadubrov.com article, "Kernmechanismen" Eq. 3; the knowledge
                 page's HC update equation.
  * mhc_projection -- the normalised projection h of the same page's rmsnorm and
                 projection equations (what the training forward saves for the backward).
  * amax_gain -- the Amax Gain Magnitude of composite residual maps ("DeepSeek-V4/mhc"
                 page, stability paragraph; slavadubrov.com numpy demo).
  * mhc_backward -- reverse mode of pre + post (the chain rule through the steps above,
                 last step first; the Sinkhorn rounds recomputed from the logits).

Parity pins for every function live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mhc_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile mhc_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
           "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_sinkhorn.argtypes = [_dp, ctypes.c_int, ctypes.c_int, _dp]
            lib.oracle_sinkhorn.restype = None
            lib.oracle_mhc_pre.argtypes = [_dp, _dp, _dp, _dp, _dp,
                                           ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                           ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_double, ctypes.c_int, _dp, _dp, ctypes.c_int]
            lib.oracle_mhc_pre.restype = None
            lib.oracle_hc_pre.argtypes = [_dp, _dp, _dp, _dp, _dp,
                                          ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                          ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_double, _dp, _dp, ctypes.c_int]
            lib.oracle_hc_pre.restype = None
            lib.oracle_mhc_post.argtypes = [_dp, _dp, _dp, ctypes.c_long, ctypes.c_int,
                                            ctypes.c_int, _dp, ctypes.c_int]
            lib.oracle_mhc_post.restype = None
            lib.oracle_mhc_projection.argtypes = [_dp, _dp, ctypes.c_long, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_double, _dp, ctypes.c_int]
            lib.oracle_mhc_projection.restype = None
            lib.oracle_mhc_backward.argtypes = ([_dp] * 6 + [ctypes.c_double] * 3 +
                                                [ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_double, ctypes.c_int] + [_dp] * 9 +
                                                [ctypes.c_int])
            lib.oracle_mhc_backward.restype = None
            lib.oracle_amax_gain.argtypes = [_dp, ctypes.c_int, ctypes.c_long, ctypes.c_int, _dp]
            lib.oracle_amax_gain.restype = None
            lib.oracle_threads_used.argtypes = [ctypes.c_int]
            lib.oracle_threads_used.restype = ctypes.c_int
            _lib = lib
    return _lib


def _c(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def sinkhorn(logits, t_max: int = 20) -> np.ndarray:
    """exp(logits), then t_max rounds of column- then row-normalisation (n x n)."""
    L = _c(logits)
    n = L.shape[0]
    assert L.shape == (n, n)
    out = np.empty_like(L)
    _load().oracle_sinkhorn(_p(L), n, int(t_max), _p(out))
    return out


def mhc_pre(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res,
            eps: float = 1e-20, t_max: int = 20, nthreads: int = 1):
    """Pre stage.  X [T, n, d] -> (x_in [T, d], H [T, n*n+2n]) in fp64."""
    X = _c(X)
    T, n, d = X.shape
    m = n * n + 2 * n
    phi = _c(phi)
    assert phi.shape == (n * d, m), phi.shape
    b_pre, b_post, b_res = _c(b_pre).reshape(n), _c(b_post).reshape(n), _c(b_res).reshape(n * n)
    x_in = np.empty((T, d), np.float64)
    H = np.empty((T, m), np.float64)
    _load().oracle_mhc_pre(_p(X), _p(phi), _p(b_pre), _p(b_post), _p(b_res),
                           float(alpha_pre), float(alpha_post), float(alpha_res),
                           T, n, d, float(eps), int(t_max), _p(x_in), _p(H), int(nthreads))
    return x_in, H


def hc_pre(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res,
           eps: float = 1e-20, nthreads: int = 1):
    """HC pre stage (unconstrained maps: bias + alpha tanh(h), no Sinkhorn).
    X [T, n, d] -> (x_in [T, d], H [T, n*n+2n]) in fp64."""
    X = _c(X)
    T, n, d = X.shape
    m = n * n + 2 * n
    phi = _c(phi)
    assert phi.shape == (n * d, m), phi.shape
    b_pre, b_post, b_res = _c(b_pre).reshape(n), _c(b_post).reshape(n), _c(b_res).reshape(n * n)
    x_in = np.empty((T, d), np.float64)
    H = np.empty((T, m), np.float64)
    _load().oracle_hc_pre(_p(X), _p(phi), _p(b_pre), _p(b_post), _p(b_res),
                          float(alpha_pre), float(alpha_post), float(alpha_res),
                          T, n, d, float(eps), _p(x_in), _p(H), int(nthreads))
    return x_in, H


def mhc_post(X, F_out, H, nthreads: int = 1) -> np.ndarray:
    """Post stage.  X [T, n, d], F_out [T, d], H [T, m] -> X' [T, n, d] in fp64."""
    X, F_out, H = _c(X), _c(F_out), _c(H)
    T, n, d = X.shape
    assert F_out.shape == (T, d) and H.shape == (T, n * n + 2 * n)
    out = np.empty_like(X)
    _load().oracle_mhc_post(_p(X), _p(F_out), _p(H), T, n, d, _p(out), int(nthreads))
    return out


def mhc_projection(X, phi, eps: float = 1e-20, nthreads: int = 1) -> np.ndarray:
    """h = RMSNorm(vec X_t) . phi for every token: X [T, n, d] -> h [T, n*n+2n] in fp64."""
    X, phi = _c(X), _c(phi)
    T, n, d = X.shape
    m = n * n + 2 * n
    assert phi.shape == (n * d, m), phi.shape
    h = np.empty((T, m), np.float64)
    _load().oracle_mhc_projection(_p(X), _p(phi), T, n, d, float(eps), _p(h), int(nthreads))
    return h


def mhc_backward(X, F_out, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res,
                 dX_out, dx_in, eps: float = 1e-20, t_max: int = 20, nthreads: int = 1) -> dict:
    """Gradients of L = <dX_out, X'> + <dx_in, x_in> with respect to every input of pre +
    post, in fp64: dict with dX [T,n,d], dF_out [T,d], dphi [n*d,m], db_pre [n],
    db_post [n], db_res [n,n] and dalpha [3] = (pre, post, res), the alpha arguments' order."""
    X, F_out, phi = _c(X), _c(F_out), _c(phi)
    T, n, d = X.shape
    m = n * n + 2 * n
    assert F_out.shape == (T, d) and phi.shape == (n * d, m)
    dX_out, dx_in = _c(dX_out), _c(dx_in)
    assert dX_out.shape == (T, n, d) and dx_in.shape == (T, d)
    b_pre, b_post, b_res = _c(b_pre).reshape(n), _c(b_post).reshape(n), _c(b_res).reshape(n * n)
    out = dict(dX=np.empty((T, n, d)), dF_out=np.empty((T, d)), dphi=np.empty((n * d, m)),
               db_pre=np.empty(n), db_post=np.empty(n), db_res=np.empty(n * n), dalpha=np.empty(3))
    _load().oracle_mhc_backward(_p(X), _p(F_out), _p(phi), _p(b_pre), _p(b_post), _p(b_res),
                                float(alpha_pre), float(alpha_post), float(alpha_res),
                                T, n, d, float(eps), int(t_max), _p(dX_out), _p(dx_in),
                                _p(out["dX"]), _p(out["dF_out"]), _p(out["dphi"]),
                                _p(out["db_pre"]), _p(out["db_post"]), _p(out["db_res"]),
                                _p(out["dalpha"]), int(nthreads))
    out["db_res"] = out["db_res"].reshape(n, n)
    return out


def amax_gain(Hs) -> np.ndarray:
    """Hs [L, T, n*n+2n] (L layers' coefficient rows) -> gain [L, T, 2]: the largest absolute
    row sum (forward) and column sum (backward) of C_l = H_res,l ... H_res,1, every l."""
    Hs = _c(Hs)
    L, T, m = Hs.shape
    n = int(round((-2 + np.sqrt(4 + 4 * m)) / 2))
    assert n * n + 2 * n == m and n <= 8, m
    g = np.empty((L, T, 2), np.float64)
    _load().oracle_amax_gain(_p(Hs), L, T, n, _p(g))
    return g


def threads_used(nthreads: int) -> int:
    """How many OpenMP threads a request of `nthreads` actually gets."""
    return int(_load().oracle_threads_used(int(nthreads)))


def split_H(H: np.ndarray, n: int):
    """Split coefficient rows [.., m] into (H_pre [..,n], H_res [..,n,n], H_post [..,n])."""
    H = np.asarray(H)
    lead = H.shape[:-1]
    return (H[..., :n], H[..., n:n + n * n].reshape(*lead, n, n), H[..., n + n * n:])
