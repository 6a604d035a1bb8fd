"""Failure detection of the tensor-core pre kernel and of the backward's tensor-core step,
without a GPU fault.

Every wait of the kernel (between its warps and between the CTAs of a cluster) is bounded
in time; a wait that runs out sets a bit in the device status word and makes the kernel
drain its own copies in flight and return.  The test hook mhc_debug_pre_stop_after makes
every cluster stop loading X at the same tile boundary, so all earlier tiles complete and
nothing is left in flight, and the waits for the tiles never loaded run into a short limit.
The test checks that the status word reports it, that the context stays usable, and that
the next normal call is correct against the oracle.  mhc_debug_backward_stop_after does the
same for the backward's dX / dphi step at a 64-token stage boundary of every CTA."""
import numpy as np
import pytest

from mhc_hyper_connections_b200 import workloads as wl

from _parity import check_against_oracle, run_gpu, run_oracle, torch_inputs

torch = pytest.importorskip("torch")
mhc = pytest.importorskip("mhc_hyper_connections_b200")

pytestmark = pytest.mark.gpu


def _tc_available(w):
    return mhc.mhc_pre_path_for(w.T, w.n, w.d, 1) == mhc.PRE_CLUSTER_TC


@pytest.fixture
def restore_hook():
    yield
    mhc.mhc_debug_pre_stop_after(-1, 1_000_000)


def test_expired_waits_are_reported_and_the_next_call_is_clean(restore_hook):
    w = wl.make_inputs(T=64 * 7 * 5, n=4, d=1024, dtype="bf16", seed=61)
    if not _tc_available(w):
        pytest.skip("no tensor-core pre path on this device")
    t = torch_inputs(w)
    s = w.scalars()
    assert mhc.mhc_device_status() == 0
    x_in = torch.zeros(w.T, w.d, dtype=torch.bfloat16, device="cuda")
    H = torch.zeros(w.T, w.m, device="cuda")
    mhc.mhc_debug_pre_stop_after(2, 50_000)        # stop after 2 tiles per cluster; 50 ms waits
    mhc.mhc_pre_with_path(t["X"], t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"],
                          s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"], x_in, H,
                          path=mhc.PRE_CLUSTER_TC)
    torch.cuda.synchronize()                        # the kernel returned: the context is usable
    code = mhc.mhc_device_status()
    assert code != 0
    assert mhc.mhc_device_status() == 0             # read-and-clear
    # the tiles before the stop were finished: x_in is written for them, not for the rest
    ref = run_oracle(w)
    done = (x_in.float().abs().sum(dim=1) > 0).cpu().numpy()
    assert done.any() and not done.all()
    mhc.mhc_debug_pre_stop_after(-1, 1_000_000)
    check_against_oracle(w, run_gpu(w, mhc.PRE_CLUSTER_TC, inputs=t), ref, "after expired waits")
    assert mhc.mhc_device_status() == 0


def test_stop_beyond_the_last_tile_changes_nothing(restore_hook):
    w = wl.make_inputs(T=300, n=4, d=2048, dtype="bf16", seed=62)
    if not _tc_available(w):
        pytest.skip("no tensor-core pre path on this device")
    ref = run_oracle(w)
    mhc.mhc_debug_pre_stop_after(1000, 50_000)
    check_against_oracle(w, run_gpu(w, mhc.PRE_CLUSTER_TC), ref, "stop past the end")
    assert mhc.mhc_device_status() == 0


# ---- the backward's tensor-core dX / dphi step

@pytest.fixture
def restore_backward_hook():
    yield
    mhc.mhc_debug_backward_stop_after(-1, 1_000_000)


def _backward_case():
    # T = 2048, d = 4096: 64 channel slices x 2 token groups of 1024, 16 stages of 64 tokens
    # per CTA on the tensor-core step
    import test_backward_gpu as tb
    w = wl.make_inputs(T=2048, n=4, d=4096, dtype="bf16", seed=63, alpha=0.3)
    dY, dx = tb._upstream(w, 64)
    return tb, w, dY, dx


def test_backward_expired_waits_are_reported_and_the_next_call_is_clean(restore_backward_hook):
    tb, w, dY, dx = _backward_case()
    t = torch_inputs(w)
    s = w.scalars()
    X, F = t["X"], t["F"]
    x_in = torch.empty(w.T, w.d, dtype=X.dtype, device="cuda")
    H = torch.empty(w.T, w.m, device="cuda")
    h = torch.empty(w.T, w.m, device="cuda")
    mhc.mhc_pre_train(X, t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"], s["alpha_post"],
                      s["alpha_res"], s["eps"], s["t_max"], x_in, H, h)
    torch.cuda.synchronize()
    assert mhc.mhc_device_status() == 0
    dX = torch.zeros_like(X)
    out = dict(dF_out=torch.empty_like(F), dphi=torch.empty(w.n * w.d, w.m, device="cuda"),
               db_pre=torch.empty(w.n, device="cuda"), db_post=torch.empty(w.n, device="cuda"),
               db_res=torch.empty(w.n, w.n, device="cuda"), dalpha=torch.empty(3, device="cuda"))
    ws = torch.empty(mhc.mhc_backward_workspace_bytes(w.T, w.n, w.d), dtype=torch.uint8, device="cuda")
    mhc.mhc_debug_backward_stop_after(2, 50_000)   # stop after 2 stages per CTA; 50 ms waits
    mhc.mhc_backward(X, F, t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"], s["alpha_post"],
                     s["alpha_res"], s["eps"], s["t_max"], H, h, tb._dev(dY), tb._dev(dx), dX, out["dF_out"],
                     out["dphi"], out["db_pre"], out["db_post"], out["db_res"], out["dalpha"], ws)
    torch.cuda.synchronize()                        # the step returned: the context is usable
    code = mhc.mhc_device_status()
    assert code >> 24 != 0                          # the backward step's bits
    assert mhc.mhc_device_status() == 0             # read-and-clear
    # the two stages before the stop were finished in both token groups: dX is written for
    # tokens 0-127 and 1024-1151, not for the others
    done = (dX.float().abs().sum(dim=(1, 2)) > 0).cpu().numpy()
    first = np.zeros(w.T, dtype=bool)
    first[0:128] = first[1024:1152] = True
    assert done[first].all() and not done[~first].any()
    mhc.mhc_debug_backward_stop_after(-1, 1_000_000)
    tb.check(w, tb.run_gpu(w, dY, dx), tb.run_oracle(w, dY, dx, nthreads=16), "after expired waits")
    assert mhc.mhc_device_status() == 0


def test_backward_stop_beyond_the_last_stage_changes_nothing(restore_backward_hook):
    tb, w, dY, dx = _backward_case()
    ref = tb.run_oracle(w, dY, dx, nthreads=16)
    mhc.mhc_debug_backward_stop_after(1000, 50_000)
    tb.check(w, tb.run_gpu(w, dY, dx), ref, "stop past the end")
    assert mhc.mhc_device_status() == 0
