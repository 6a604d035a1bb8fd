"""Out-of-bounds write checks with guard regions, the stand-in for a memory sanitizer.

Every output of mhc_pre, mhc_pre_train, mhc_post, mhc_backward (its workspace included)
and mhc_amax_gain is a view with GUARD bytes of a fixed pattern before and after it.
After the call both guards must be intact, and the outputs must equal, bit for bit, those
of the same call on plain tensors (every kernel here is deterministic).  The shapes are
those of the parity tests: ragged token tails, odd d, all three pre paths (the two-pass
tensor-core path uses x_in as scratch before writing it) and both post kernels."""
import numpy as np
import pytest

from mhc_hyper_connections_b200 import workloads as wl

from _canary import guarded_empty, guards_intact
from _parity import torch_inputs

torch = pytest.importorskip("torch")
mhc = pytest.importorskip("mhc_hyper_connections_b200")

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _outputs(spec, guarded):
    """spec: name -> (shape, dtype).  Returns (views, buffers); buffers is empty when plain."""
    views, bufs = {}, {}
    for k, (shape, dt) in spec.items():
        if guarded:
            bufs[k], views[k] = guarded_empty(shape, dt, DEV)
        else:
            views[k] = torch.empty(*shape, dtype=dt, device=DEV)
    return views, bufs


def _same_and_intact(plain, guarded, bufs):
    torch.cuda.synchronize()
    for k, b in bufs.items():
        assert guards_intact(b), f"{k}: a kernel wrote outside this output"
    for k in plain:
        if k == "ws":
            continue
        assert torch.equal(plain[k], guarded[k]), f"{k}: differs from the unguarded call"


@pytest.mark.parametrize("T,n,d,dt", [(1, 4, 64, "bf16"), (17, 4, 1024, "bf16"), (19, 3, 40, "f32"),
                                      (9, 8, 64, "f32"), (3, 4, 37, "bf16"), (100, 4, 2048, "bf16"),
                                      (130, 4, 4096, "bf16"), (40, 1, 1024, "bf16"), (77, 4, 2560, "bf16"),
                                      (2000, 8, 4096, "bf16"), (400, 4, 8192, "bf16")])
def test_forward_writes_stay_inside_their_outputs(T, n, d, dt):
    w = wl.make_inputs(T=T, n=n, d=d, dtype=dt, seed=T + n + d, outlier_frac=0.01)
    t = torch_inputs(w, device=DEV)
    X, s = t["X"], w.scalars()
    spec = dict(x_in=((T, d), X.dtype), H=((T, w.m), torch.float32), Y=((T, n, d), X.dtype))
    res = []
    for guarded in (False, True):
        o, bufs = _outputs(spec, guarded)
        mhc.mhc_pre(X, t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"], s["alpha_post"],
                    s["alpha_res"], s["eps"], s["t_max"], o["x_in"], o["H"])
        mhc.mhc_post(X, t["F"], o["H"], o["Y"])
        res.append((o, bufs))
    _same_and_intact(res[0][0], res[1][0], res[1][1])


@pytest.mark.parametrize("T,n,d,dt", [(100, 3, 136, "bf16"), (33, 2, 24, "f32"), (300, 1, 1024, "bf16"),
                                      (700, 4, 512, "bf16"), (129, 3, 192, "bf16"), (65, 2, 64, "bf16")])
def test_training_writes_stay_inside_their_outputs(T, n, d, dt):
    w = wl.make_inputs(T=T, n=n, d=d, dtype=dt, seed=2 * T + d, alpha=0.3)
    t = torch_inputs(w, device=DEV)
    X, F, s, m = t["X"], t["F"], w.scalars(), w.m
    rng = np.random.default_rng(T + n)
    up = [rng.standard_normal(sh, dtype=np.float32) for sh in ((T, n, d), (T, d))]
    dY, dx = (torch.from_numpy(a).to(DEV).to(X.dtype) for a in up)
    f32 = torch.float32
    need = mhc.mhc_backward_workspace_bytes(T, n, d)
    spec = dict(x_in=((T, d), X.dtype), H=((T, m), f32), h=((T, m), f32), dX=((T, n, d), X.dtype),
                dF_out=((T, d), X.dtype), dphi=((n * d, m), f32), db_pre=((n,), f32), db_post=((n,), f32),
                db_res=((n, n), f32), dalpha=((3,), f32), ws=((need,), torch.uint8))
    sa = (s["alpha_pre"], s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"])
    res = []
    for guarded in (False, True):
        o, bufs = _outputs(spec, guarded)
        mhc.mhc_pre_train(X, t["phi"], t["b_pre"], t["b_post"], t["b_res"], *sa, o["x_in"], o["H"], o["h"])
        mhc.mhc_backward(X, F, t["phi"], t["b_pre"], t["b_post"], t["b_res"], *sa, o["H"], o["h"], dY, dx,
                         o["dX"], o["dF_out"], o["dphi"], o["db_pre"], o["db_post"], o["db_res"], o["dalpha"],
                         o["ws"])
        res.append((o, bufs))
    _same_and_intact(res[0][0], res[1][0], res[1][1])


def test_amax_gain_writes_stay_inside_its_output():
    Hs = torch.from_numpy(np.random.default_rng(7).normal(size=(3, 50, 24)).astype(np.float32)).to(DEV)
    res = []
    for guarded in (False, True):
        o, bufs = _outputs(dict(gain=((3, 50, 2), torch.float32)), guarded)
        mhc.mhc_amax_gain(Hs, o["gain"])
        res.append((o, bufs))
    _same_and_intact(res[0][0], res[1][0], res[1][1])
