"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle on the same
seeded inputs -- element by element on every token of every workload (the large ones in
token chunks on all host cores), plus size-independent properties at the full sizes."""
import os

import numpy as np
import pytest

import oracle
from mhc_hyper_connections_b200 import workloads as wl

from _parity import check_against_oracle, run_gpu, run_oracle, to_f64, torch_inputs

torch = pytest.importorskip("torch")
mhc = pytest.importorskip("mhc_hyper_connections_b200")

pytestmark = pytest.mark.gpu


def _paths(w):
    """Every pre path that can run this workload on this device."""
    dt = 1 if w.dtype == "bf16" else 0
    return [p for p in (mhc.PRE_GENERIC, mhc.PRE_CLUSTER_TC, mhc.PRE_TWO_PASS_TC)
            if mhc.mhc_pre_path_ok(w.T, w.n, w.d, dt, p)]


def test_library_is_the_one_in_tree():
    import os
    lib = mhc.load_library()
    assert os.path.dirname(mhc.library_path()) == os.path.dirname(mhc.__file__)
    assert lib is not None


def test_tiny_f32_config_full():
    w = wl.make_config("tiny_f32_T64_n4_d64")
    ref = run_oracle(w)
    for p in _paths(w):
        check_against_oracle(w, run_gpu(w, p), ref, f"tiny path{p}")


def test_bf16_d1024_config_full():
    w = wl.make_config("bf16_T4096_n4_d1024")
    ref = run_oracle(w)
    for p in _paths(w):
        check_against_oracle(w, run_gpu(w, p), ref, f"d1024 path{p}")


def _full_size_properties(w, gpu, inputs):
    """Properties that hold for every token at any size (checked on the GPU in fp32)."""
    x_in, H, Y = gpu
    n = w.n
    Hp, Hr, Hq = H[:, :n], H[:, n:n + n * n].reshape(-1, n, n), H[:, n + n * n:]
    assert torch.isfinite(H).all()
    assert ((Hp > 0) & (Hp < 1)).all() and ((Hq > 0) & (Hq < 2)).all() and (Hr > 0).all()
    assert (Hr.sum(dim=2) - 1).abs().max().item() <= 1e-5       # final step normalises rows
    X = inputs["X"].float()
    F = inputs["F"].float()
    ref_x = torch.einsum("ti,tic->tc", Hp, X)
    S_x = torch.einsum("ti,tic->tc", Hp.abs(), X.abs())
    assert ((x_in.float() - ref_x).abs() <= 2 ** -8 * ref_x.abs() + 1e-5 * S_x).all()
    for i in range(n):   # stream by stream to bound memory
        ref_y = torch.einsum("tj,tjc->tc", Hr[:, i], X) + Hq[:, i:i + 1] * F
        S_y = torch.einsum("tj,tjc->tc", Hr[:, i].abs(), X.abs()) + Hq[:, i:i + 1].abs() * F.abs()
        assert ((Y[:, i].float() - ref_y).abs() <= 2 ** -8 * ref_y.abs() + 1e-5 * S_y).all()


def compare_all_tokens(w, gpu, label, chunk=1024):
    """Every token of a workload against the oracle, element by element: the oracle runs over
    consecutive token chunks (it depends on nothing across tokens) on all host cores, and each
    chunk is compared with the same rows of the GPU outputs."""
    x_in, H, Y = gpu
    worst = {}
    for c0 in range(0, w.T, chunk):
        c1 = min(w.T, c0 + chunk)
        sub = w.tokens(np.arange(c0, c1))
        errs = check_against_oracle(sub, (x_in[c0:c1], H[c0:c1], Y[c0:c1]),
                                    run_oracle(sub, nthreads=os.cpu_count() or 8),
                                    f"{label} tokens {c0}..{c1 - 1}")
        for k, v in errs.items():
            worst[k] = max(worst.get(k, 0.0), v)
    return worst


@pytest.mark.parametrize("name", ["bf16_T16384_n4_d4096_outliers", "bf16_T8192_n8_d4096"])
def test_full_size_configs_all_tokens(name):
    """The two large forward workloads, every token and every output element against the
    oracle, on every pre path the device runs for them; plus the size-independent
    properties on the GPU."""
    w = wl.make_config(name)
    inputs = torch_inputs(w)
    for p in _paths(w):
        gpu = run_gpu(w, p, inputs=inputs)
        _full_size_properties(w, gpu, inputs)
        worst = compare_all_tokens(w, gpu, f"{name} path{p}")
        assert worst["H"] <= 1e-4 and worst["x_in"] <= 2e-2 and worst["X_out"] <= 2e-2, worst
        del gpu
    torch.cuda.empty_cache()


SHAPES = [  # (T, n, d, dtype): ragged token tails, odd d, every n
    (1, 4, 64, "bf16"), (17, 4, 1024, "bf16"), (33, 1, 8, "f32"), (5, 2, 12, "bf16"),
    (19, 3, 40, "f32"), (7, 5, 24, "bf16"), (9, 8, 64, "f32"), (3, 4, 37, "bf16"),
    (100, 4, 2048, "bf16"), (50, 4, 3072, "bf16"), (31, 6, 16, "bf16"), (12, 7, 9, "f32"),
    (130, 4, 4096, "bf16"), (23, 2, 1024, "bf16"), (40, 1, 1024, "bf16"),
    # tensor-core path at channel counts off the powers of two, several tiles per cluster
    (77, 4, 2560, "bf16"), (65, 4, 5120, "bf16"), (1363, 4, 512, "bf16"), (200, 3, 1280, "bf16"),
    (129, 2, 768, "bf16"), (1000, 1, 1024, "bf16"), (64 * 7 * 3 + 17, 4, 1024, "bf16"),
    # two-pass tensor-core path: n = 5..8, and d past the cluster kernel's shared memory
    (2000, 8, 4096, "bf16"), (2100, 7, 2048, "bf16"), (1500, 6, 1536, "bf16"),
    (2100, 5, 1024, "bf16"), (400, 4, 8192, "bf16"), (350, 4, 7168, "bf16"), (300, 4, 6144, "bf16"),
    (1300, 4, 2048, "bf16"), (700, 3, 1024, "bf16"), (900, 5, 1088, "bf16"),
]


@pytest.mark.parametrize("T,n,d,dt", SHAPES)
def test_shapes(T, n, d, dt):
    w = wl.make_inputs(T=T, n=n, d=d, dtype=dt, seed=T * 131 + n * 17 + d)
    ref = run_oracle(w)
    for p in _paths(w):
        check_against_oracle(w, run_gpu(w, p), ref, f"T{T} n{n} d{d} {dt} path{p}")


def test_strong_dynamic_maps():
    """alpha = 1 makes the dynamic term dominate (later-training regime)."""
    w = wl.make_inputs(T=64, n=4, d=1024, dtype="bf16", seed=77, alpha=1.0)
    ref = run_oracle(w)
    for p in _paths(w):
        check_against_oracle(w, run_gpu(w, p), ref, f"alpha1 path{p}")


def test_zero_token_row():
    w = wl.make_inputs(T=20, n=4, d=1024, dtype="bf16", seed=5)
    w.X[3] = 0
    ref = run_oracle(w)
    for p in _paths(w):
        gpu = run_gpu(w, p)
        check_against_oracle(w, gpu, ref, f"zero-token path{p}")
        assert (gpu[0][3] == 0).all()


def test_T0_is_noop():
    w = wl.make_inputs(T=4, n=4, d=64, dtype="bf16", seed=1)
    t = torch_inputs(w)
    x_in = torch.full((0, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    H = torch.empty(0, 24, device="cuda")
    Xe = t["X"][:0]
    mhc.mhc_pre(Xe, t["phi"], t["b_pre"], t["b_post"], t["b_res"], 0.01, 0.01, 0.01, 1e-20, 20,
                x_in, H)
    mhc.mhc_post(Xe, t["F"][:0], H, torch.empty_like(Xe))
    torch.cuda.synchronize()


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_post_identity_is_bit_exact(dt):
    w = wl.make_inputs(T=37, n=4, d=256, dtype=dt, seed=9)
    t = torch_inputs(w)
    H = torch.zeros(w.T, w.m, device="cuda")
    H[:, 4:20] = torch.eye(4, device="cuda").reshape(-1)
    Y = torch.empty_like(t["X"])
    mhc.mhc_post(t["X"], t["F"], H, Y)
    torch.cuda.synchronize()
    assert torch.equal(Y, t["X"])


def test_deterministic_bitwise():
    w = wl.make_inputs(T=300, n=4, d=1024, dtype="bf16", seed=21)
    t = torch_inputs(w)
    for p in _paths(w):
        a = run_gpu(w, p, inputs=t)
        b = run_gpu(w, p, inputs=t)
        for u, v in zip(a, b):
            assert torch.equal(u, v)


def test_unaligned_buffers_take_scalar_kernels():
    """X, F_out and X_out 2 bytes off a 16-byte boundary: same results, scalar kernels."""
    w = wl.make_inputs(T=9, n=4, d=64, dtype="bf16", seed=31)
    ref = run_oracle(w)
    t = torch_inputs(w)
    Xb = torch.empty(w.T * 4 * 64 + 1, dtype=torch.bfloat16, device="cuda")
    Fb = torch.empty(w.T * 64 + 1, dtype=torch.bfloat16, device="cuda")
    Yb = torch.empty(w.T * 4 * 64 + 1, dtype=torch.bfloat16, device="cuda")
    X = Xb[1:].view(w.T, 4, 64)
    F = Fb[1:].view(w.T, 64)
    Y = Yb[1:].view(w.T, 4, 64)
    X.copy_(t["X"])
    F.copy_(t["F"])
    x_in = torch.empty(w.T, 64, dtype=torch.bfloat16, device="cuda")
    H = torch.empty(w.T, 24, device="cuda")
    s = w.scalars()
    mhc.mhc_pre(X, t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"],
                s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"], x_in, H)
    mhc.mhc_post(X, F, H, Y)
    torch.cuda.synchronize()
    check_against_oracle(w, (x_in, H, Y), ref, "unaligned")


def test_paths_agree_with_each_other():
    w = wl.make_config("bf16_T4096_n4_d1024")
    paths = _paths(w)
    if len(paths) < 2:
        pytest.skip("only one pre path on this device for this shape")
    t = torch_inputs(w)
    g = run_gpu(w, paths[0], inputs=t)
    for p in paths[1:]:
        c = run_gpu(w, p, inputs=t)
        assert (g[1] - c[1]).abs().max().item() <= 1e-5
        d = (g[0].float() - c[0].float()).abs()
        assert (d <= 2 ** -7 * g[0].float().abs() + 1e-5).all()


def test_auto_path_on_b200_shapes_is_tensor_core():
    """On a B200 the bf16 shapes with n <= 4, d a multiple of 64, n*d >= 1024 and a phi slice
    that fits shared memory run the cluster tensor-core kernel; other bf16 shapes up to n = 8
    whose x_in buffer can hold the packed phi run the two-pass tensor-core kernels; the rest
    runs the generic kernel."""
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip("not an sm_100 device")
    for n in (1, 2, 3, 4):
        for d in (1024, 2048, 2560, 3072, 4096, 5120):
            assert mhc.mhc_pre_path_for(16384, n, d, 1) == mhc.PRE_CLUSTER_TC, (n, d)
    assert mhc.mhc_pre_path_for(16384, 4, 512, 1) == mhc.PRE_CLUSTER_TC       # n*d = 2048
    assert mhc.mhc_pre_path_for(16384, 4, 4096, 0) == mhc.PRE_GENERIC         # fp32 storage
    assert mhc.mhc_pre_path_for(8192, 8, 4096, 1) == mhc.PRE_TWO_PASS_TC      # n = 8
    for d in (6144, 7168, 8192):                                             # large d at n = 4
        assert mhc.mhc_pre_path_for(16384, 4, d, 1) == mhc.PRE_TWO_PASS_TC, d
    assert mhc.mhc_pre_path_for(100, 8, 4096, 1) == mhc.PRE_GENERIC           # x_in too small for scratch
    assert mhc.mhc_pre_path_for(16384, 4, 4100, 1) == mhc.PRE_GENERIC         # d % 64 != 0
    assert mhc.mhc_pre_path_for(16384, 2, 256, 1) == mhc.PRE_TWO_PASS_TC      # n*d = 512
    assert mhc.mhc_pre_path_for(16384, 1, 192, 1) == mhc.PRE_GENERIC          # n*d < 256


def test_device_status_clean_after_runs():
    """Every bounded wait of the tensor-core kernel completed in the runs above."""
    w = wl.make_inputs(T=77, n=4, d=2048, dtype="bf16", seed=8)
    run_gpu(w)
    assert mhc.mhc_device_status() == 0


def test_tensor_core_path_rejects_what_it_cannot_run():
    w = wl.make_inputs(T=8, n=4, d=64, dtype="bf16", seed=2)
    t = torch_inputs(w)
    x_in = torch.empty(8, 64, dtype=torch.bfloat16, device="cuda")
    H = torch.empty(8, 24, device="cuda")
    for path in (mhc.PRE_CLUSTER_TC,):
        with pytest.raises(mhc.MhcError, match="UNSUPPORTED"):
            mhc.mhc_pre_with_path(t["X"], t["phi"], t["b_pre"], t["b_post"], t["b_res"], 0.01,
                                  0.01, 0.01, 1e-20, 20, x_in, H, path=path)


def test_single_atom_tiles_after_dirty_tmem():
    """n = 1, d = 1024 gives one K atom per CTA, so all but one of the tensor-core kernel's
    MMA accumulators receive no MMA; they must not be added in.  A launch at n = 4 first
    leaves non-zero accumulators in TMEM on the same SMs."""
    dirty = wl.make_inputs(T=2048, n=4, d=4096, dtype="bf16", seed=41)
    w = wl.make_inputs(T=300, n=1, d=1024, dtype="bf16", seed=42)
    ref = run_oracle(w)
    for p in _paths(w)[1:]:
        for _ in range(2):
            run_gpu(dirty, p)
            check_against_oracle(w, run_gpu(w, p), ref, f"after dirty TMEM path{p}")
