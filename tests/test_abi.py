"""The C-ABI library loads, exports every symbol include/mhc.h declares, and rejects bad
arguments on the host (status codes, no launch).  No compute call runs here: every call
below fails validation before the library touches CUDA."""
import ctypes
import os
import re

import pytest

import mhc_hyper_connections_b200 as mhc
from mhc_hyper_connections_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mbuild.build()
    return mhc.load_library()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "mhc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(mhc_\w+)\s*\(", src))


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert declared == set(mhc.EXPORTED_SYMBOLS)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(9):
        s = lib.mhc_status_string(code)
        assert s and s.decode() != "unknown status"
    assert lib.mhc_status_string(99).decode() == "unknown status"
    assert lib.mhc_last_error().decode() == ""


# fake, never-dereferenced addresses: validation rejects before any CUDA call
A = 0x10000000


def _pre(lib, X=A, phi=A + 0x1000000, bp=A + 0x2000000, bq=A + 0x2000100, br=A + 0x2000200,
         T=4, n=4, d=64, t_max=20, dt=1, x_in=A + 0x3000000, H=A + 0x4000000):
    return lib.mhc_pre(X, phi, bp, bq, br, 0.01, 0.01, 0.01, T, n, d, 1e-20, t_max, dt, x_in, H, None)


def test_pre_validation(lib):
    assert _pre(lib, T=0) == 0                       # T = 0 is a no-op
    assert _pre(lib, T=0, X=0, x_in=0, H=0) == 0     # ... even with NULL buffers
    assert _pre(lib, n=0) == 2 and _pre(lib, n=9) == 2
    assert _pre(lib, d=0) == 2 and _pre(lib, T=-1) == 2
    assert _pre(lib, t_max=-1) == 2 and _pre(lib, t_max=1001) == 2
    assert _pre(lib, dt=2) == 4
    assert _pre(lib, X=0) == 1 and _pre(lib, H=0) == 1 and _pre(lib, phi=0) == 1
    assert _pre(lib, br=0) == 1
    assert _pre(lib, X=A + 1) == 3                   # bf16 needs 2-byte alignment
    assert _pre(lib, dt=0, X=A + 2) == 3             # fp32 needs 4
    assert _pre(lib, H=A + 0x4000002) == 3
    assert _pre(lib, x_in=A + 16) == 7               # x_in overlaps X
    assert _pre(lib, H=A + 0x3000010) == 7           # H overlaps x_in
    assert _pre(lib, H=A + 0x1000000) == 7           # H overlaps phi
    huge = (1 << 62) // (4 * 64)
    assert _pre(lib, T=huge) == 2                    # byte counts would overflow


def test_pre_with_path_rejects_unknown_path(lib):
    st = lib.mhc_pre_with_path(A, A + 0x1000000, A + 0x2000000, A + 0x2000100, A + 0x2000200,
                               0.01, 0.01, 0.01, 4, 4, 64, 1e-20, 20, 1, A + 0x3000000,
                               A + 0x4000000, None, 7)
    assert st == 5


def test_post_validation(lib):
    def post(X=A, F=A + 0x1000000, H=A + 0x2000000, T=4, n=4, d=64, dt=1, Y=A + 0x3000000):
        return lib.mhc_post(X, F, H, T, n, d, dt, Y, None)
    assert post(T=0) == 0
    assert post(n=0) == 2 and post(d=-3) == 2
    assert post(dt=7) == 4
    assert post(Y=0) == 1 and post(F=0) == 1
    assert post(X=A + 1) == 3
    assert post(Y=A + 64) == 7                       # X_out overlaps X
    assert post(Y=A + 0x1000000) == 7                # X_out overlaps F_out


def test_forward_host_validation(lib):
    """mhc_forward_host: every rejection happens before the library touches CUDA."""
    n, d, T, ct = 4, 64, 10, 4
    ws_need = lib.mhc_forward_host_workspace_bytes(ct, n, d, 1)
    assert ws_need > 0
    assert lib.mhc_forward_host_workspace_bytes(2 * ct, n, d, 1) > ws_need
    assert lib.mhc_forward_host_workspace_bytes(0, n, d, 1) == 0
    assert lib.mhc_forward_host_workspace_bytes(ct, 9, d, 1) == 0
    assert lib.mhc_forward_host_workspace_bytes(ct, n, d, 5) == 0
    assert lib.mhc_forward_host_workspace_bytes(1 << 40, n, d, 1) == 0   # a chunk too large

    def expect(ct, n, d, es):   # three sets of X, F_out, x_in, H, X_out, each 256-byte aligned
        up = lambda b: (b + 255) // 256 * 256
        m = n * n + 2 * n
        return 3 * (2 * up(ct * n * d * es) + 2 * up(ct * d * es) + up(ct * m * 4))
    for ct_, n_, d_, dt_, es in ((4, 4, 64, 1, 2), (1024, 4, 4096, 1, 2), (7, 3, 100, 0, 4), (1, 8, 8, 1, 2)):
        assert lib.mhc_forward_host_workspace_bytes(ct_, n_, d_, dt_) == expect(ct_, n_, d_, es)

    W = A + 0x5000000                                # device workspace (256-aligned)

    def fh(Xh=A, Fh=A + 0x1000000, phi=A + 0x6000000, bp=A + 0x7000000, bq=A + 0x7000100,
           br=A + 0x7000200, T=T, n=n, d=d, t_max=20, dt=1, xin=A + 0x2000000, Hh=A + 0x3000000,
           Yh=A + 0x4000000, ct=ct, ws=W, wsb=ws_need):
        return lib.mhc_forward_host(Xh, Fh, phi, bp, bq, br, 0.01, 0.01, 0.01, T, n, d, 1e-20,
                                    t_max, dt, xin, Hh, Yh, ct, ws, wsb, None)
    assert fh(T=0) == 0 and fh(T=0, Xh=0, ws=0) == 0   # no tokens: nothing to do
    assert fh(n=9) == 2 and fh(d=0) == 2 and fh(t_max=1001) == 2
    assert fh(ct=0) == 2 and fh(ct=-5) == 2
    assert fh(dt=3) == 4
    assert fh(Xh=0) == 1 and fh(Yh=0) == 1 and fh(ws=0) == 1 and fh(br=0) == 1
    assert fh(Xh=A + 1) == 3 and fh(Hh=A + 0x3000002) == 3
    assert fh(ws=W + 16) == 3                        # the workspace needs 256-byte alignment
    assert fh(wsb=ws_need - 1) == 8
    assert fh(ct=100) == 8                           # a chunk above T takes all T = 10 tokens
    assert fh(xin=A + 64) == 7                       # x_in_h overlaps X_h
    assert fh(Yh=A + 0x1000000) == 7                 # X_out_h overlaps F_out_h
    assert fh(Hh=A + 0x2000000) == 7                 # H_h overlaps x_in_h
    assert fh(phi=W + 256) == 7                      # the workspace holds phi


def test_binding_refuses_host_tensors():
    torch = pytest.importorskip("torch")
    X = torch.zeros(2, 4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mhc.mhc_post(X, torch.zeros(2, 8, dtype=torch.bfloat16), torch.zeros(2, 24),
                     torch.zeros_like(X))


def test_path_query_on_cpu_host(lib):
    # With no usable GPU the query answers the generic path and launches nothing.
    assert lib.mhc_pre_path_for(16, 4, 64, 0) == mhc.PRE_GENERIC


def _bwd(lib, X=A, F=A + 0x1000000, phi=A + 0x2000000, bp=A + 0x3000000, bq=A + 0x3000100,
         br=A + 0x3000200, H=A + 0x4000000, h=A + 0x5000000, T=4, n=4, d=64, t_max=20, dt=1,
         dY=A + 0x6000000, dx=A + 0x7000000, dX=A + 0x8000000, dF=A + 0x9000000,
         dphi=A + 0xA000000, dbp=A + 0xB000000, dbq=A + 0xB000100, dbr=A + 0xB000200,
         dal=A + 0xB000400, ws=A + 0xC000000, wsb=1 << 24):
    return lib.mhc_backward(X, F, phi, bp, bq, br, 0.01, 0.01, 0.01, H, h, T, n, d, 1e-20, t_max,
                            dt, dY, dx, dX, dF, dphi, dbp, dbq, dbr, dal, ws, wsb, None)


def test_backward_validation(lib):
    assert lib.mhc_backward_workspace_bytes(4, 4, 64) > 0
    assert lib.mhc_backward_workspace_bytes(4, 5, 64) == 0          # n > 4: not supported
    assert _bwd(lib, n=5) == 5 and _bwd(lib, n=0) == 2
    assert _bwd(lib, t_max=-1) == 2 and _bwd(lib, dt=3) == 4
    assert _bwd(lib, X=0) == 1 and _bwd(lib, ws=0) == 1 and _bwd(lib, phi=0) == 1
    assert _bwd(lib, dal=0) == 1
    assert _bwd(lib, X=A + 2) == 3                   # 16-byte alignment for the vector loads
    assert _bwd(lib, d=60) == 3                      # 120-byte rows are not 16-byte multiples
    assert _bwd(lib, ws=A + 0xC000010) == 3          # workspace: 256-byte alignment
    need = lib.mhc_backward_workspace_bytes(4, 4, 64)
    assert _bwd(lib, wsb=need - 1) == 8
    assert _bwd(lib, dX=A + 64) == 7                 # dX overlaps X
    assert _bwd(lib, dphi=A + 0xC000000) == 7        # dphi overlaps the workspace
    assert _bwd(lib, dF=A + 0x6000000) == 7          # dF_out overlaps dX_out


def test_pre_train_validation(lib):
    def pre_train(h=A + 0x5000000, H=A + 0x4000000, T=4):
        return lib.mhc_pre_train(A, A + 0x1000000, A + 0x2000000, A + 0x2000100, A + 0x2000200,
                                 0.01, 0.01, 0.01, T, 4, 64, 1e-20, 20, 1, A + 0x3000000, H, h, None)
    assert pre_train(T=0) == 0
    assert pre_train(h=0) == 1
    assert pre_train(h=A + 0x5000002) == 3
    assert pre_train(h=A + 0x4000000) == 7           # h overlaps H


def test_amax_gain_validation(lib):
    assert lib.mhc_amax_gain(A, 0, 5, 4, A + 0x1000000, None) == 0      # L = 0: nothing to do
    assert lib.mhc_amax_gain(A, 3, 0, 4, A + 0x1000000, None) == 0      # T = 0
    assert lib.mhc_amax_gain(A, 3, 5, 9, A + 0x1000000, None) == 2
    assert lib.mhc_amax_gain(A, -1, 5, 4, A + 0x1000000, None) == 2
    assert lib.mhc_amax_gain(0, 3, 5, 4, A + 0x1000000, None) == 1
    assert lib.mhc_amax_gain(A, 3, 5, 4, A + 2, None) == 3
    assert lib.mhc_amax_gain(A, 3, 5, 4, A + 64, None) == 7             # gain overlaps H_layers


def test_debug_stop_hook_validation(lib):
    """The failure-path test hook checks its wait limit on the host; the default setting
    (never stop, 1 s waits) is restored at the end."""
    assert lib.mhc_debug_pre_stop_after(-1, 999) == 2
    assert lib.mhc_debug_pre_stop_after(3, 10_000_001) == 2
    assert lib.mhc_debug_pre_stop_after(-1, 1_000_000) == 0
    assert lib.mhc_debug_backward_stop_after(-1, 999) == 2
    assert lib.mhc_debug_backward_stop_after(3, 10_000_001) == 2
    assert lib.mhc_debug_backward_stop_after(-1, 1_000_000) == 0
