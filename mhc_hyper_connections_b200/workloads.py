"""Seeded synthetic inputs for the mHC pre/post path.

This module holds no arithmetic of the method: it only draws random numbers and rounds
them to the storage type.  Both the CUDA path's tests/benchmark and the CPU oracle take
their inputs from here, so the two sides see bit-identical data.

Recipe (shapes and distributions of the workloads the mHC pages describe; n = 4 streams,
alpha = 0.01, t_max = 20, RMSNorm eps = 1e-20 as on the "DeepSeek-V4/mhc" page):
  * X ~ N(0, 1) [T, n, d], F_out ~ N(0, 1) [T, d], drawn in fp32 with numpy PCG64 and
    rounded to bf16 (round to nearest even) for the bf16 workloads;
  * phi ~ N(0, 1/(n d)) [n d, n^2 + 2n] in fp32 (variance 1/(n d));
  * b_pre = b_post = 0, b_res = 4 I + N(0, 0.1) (variance 0.1), fp32;
  * optional outlier channels: ceil(frac * d) channel indices drawn by a seeded
    permutation, and X[:, :, c], F_out[:, c] scaled by 20 before rounding.
Draw order within one seed: X, F_out, phi, b_res noise, outlier permutation.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

ALPHA = 0.01
EPS = 1e-20
T_MAX = 20


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round to nearest even (NaN kept quiet)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = np.uint16(0x7FC0)
    return r


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp32 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Workload:
    name: str
    T: int
    n: int
    d: int
    dtype: str                 # "bf16" or "f32": storage type of X, F_out, x_in, X'
    X: np.ndarray              # [T, n, d]  uint16 bf16 bits or float32
    F_out: np.ndarray          # [T, d]
    phi: np.ndarray            # [n d, m] float32
    b_pre: np.ndarray          # [n] float32
    b_post: np.ndarray         # [n] float32
    b_res: np.ndarray          # [n, n] float32
    alpha_pre: float = ALPHA
    alpha_post: float = ALPHA
    alpha_res: float = ALPHA
    eps: float = EPS
    t_max: int = T_MAX
    outlier_channels: np.ndarray | None = None

    @property
    def m(self) -> int:
        return self.n * self.n + 2 * self.n

    def values(self, arr: np.ndarray) -> np.ndarray:
        """The exact fp64 values an array of this workload stores."""
        if arr.dtype == np.uint16:
            return bf16_bits_to_f32(arr).astype(np.float64)
        return np.asarray(arr, dtype=np.float64)

    def scalars(self) -> dict:
        """alpha / eps as the fp32 values the GPU receives, widened exactly to fp64."""
        f = lambda v: float(np.float32(v))
        return dict(alpha_pre=f(self.alpha_pre), alpha_post=f(self.alpha_post),
                    alpha_res=f(self.alpha_res), eps=f(self.eps), t_max=self.t_max)

    def tokens(self, idx) -> "Workload":
        """Sub-workload holding only the tokens `idx` (same parameters)."""
        idx = np.asarray(idx)
        return dataclasses.replace(self, T=int(idx.size), X=self.X[idx], F_out=self.F_out[idx],
                                   name=f"{self.name}[{idx.size} tokens]")


def make_inputs(T: int, n: int, d: int, dtype: str = "bf16", seed: int = 0,
                outlier_frac: float = 0.0, alpha: float = ALPHA, b_res_diag: float = 4.0,
                b_res_var: float = 0.1, name: str | None = None) -> Workload:
    if dtype not in ("bf16", "f32"):
        raise ValueError(dtype)
    rng = np.random.default_rng(seed)
    m = n * n + 2 * n
    X = rng.standard_normal((T, n, d), dtype=np.float32)
    F = rng.standard_normal((T, d), dtype=np.float32)
    phi = rng.standard_normal((n * d, m), dtype=np.float32) * np.float32(1.0 / math.sqrt(n * d))
    b_res = (b_res_diag * np.eye(n) + rng.standard_normal((n, n)) * math.sqrt(b_res_var)).astype(np.float32)
    ch = None
    if outlier_frac > 0:
        k = int(math.ceil(outlier_frac * d))
        ch = np.sort(rng.permutation(d)[:k])
        X[:, :, ch] *= np.float32(20.0)
        F[:, ch] *= np.float32(20.0)
    if dtype == "bf16":
        X, F = bf16_round_bits(X), bf16_round_bits(F)
    return Workload(name=name or f"T{T}_n{n}_d{d}_{dtype}_s{seed}", T=T, n=n, d=d, dtype=dtype,
                    X=X, F_out=F, phi=phi.astype(np.float32), b_pre=np.zeros(n, np.float32),
                    b_post=np.zeros(n, np.float32), b_res=b_res, alpha_pre=alpha,
                    alpha_post=alpha, alpha_res=alpha, outlier_channels=ch)


# The four forward workloads (and one extra shape): sizes, storage type, seed and outlier structure.
CONFIGS = {
    "tiny_f32_T64_n4_d64": dict(T=64, n=4, d=64, dtype="f32", seed=0),
    "bf16_T4096_n4_d1024": dict(T=4096, n=4, d=1024, dtype="bf16", seed=1),
    "bf16_T16384_n4_d4096_outliers": dict(T=16384, n=4, d=4096, dtype="bf16", seed=2,
                                          outlier_frac=0.01),
    "bf16_T8192_n8_d4096": dict(T=8192, n=8, d=4096, dtype="bf16", seed=3),
    # not one of the four: the hidden size of the 27B model in the "DeepSeek-V4/mhc" model
    # table, for a bench figure of that shape
    "bf16_T16384_n4_d2560": dict(T=16384, n=4, d=2560, dtype="bf16", seed=4),
}

HEADLINE = "bf16_T16384_n4_d4096_outliers"


def make_config(name: str) -> Workload:
    return make_inputs(name=name, **CONFIGS[name])
