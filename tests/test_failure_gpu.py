"""Failure detection of the tensor-core pre kernel, without a GPU fault.

Every wait of the kernel (between its warps and between the CTAs of a cluster) is bounded
in time; a wait that runs out sets a bit in the device status word and makes the kernel
drain its own copies in flight and return.  The test hook mhc_debug_pre_stop_after makes
every cluster stop loading X at the same tile boundary, so all earlier tiles complete and
nothing is left in flight, and the waits for the tiles never loaded run into a short limit.
The test checks that the status word reports it, that the context stays usable, and that
the next normal call is correct against the oracle."""
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
