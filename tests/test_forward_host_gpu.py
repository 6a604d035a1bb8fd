"""mhc_forward_host (pre then post on activations in host memory, chunked through three
device buffer sets with the copies overlapped) against the device entry points and the oracle.

Every output of a token depends on that token alone, so the host path must give, bit for bit,
what mhc_pre and mhc_post give when called on the same chunks. Where each chunk takes the
whole batch's kernel path, that is also the whole-batch result. The oracle check covers the
first and last chunk, including a ragged tail."""
import numpy as np
import pytest

import mhc_hyper_connections_b200 as mhc
from mhc_hyper_connections_b200 import workloads as wl

from _parity import check_against_oracle, run_gpu, run_oracle, torch_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _host_buffers(w, t, pinned=True):
    X = t["X"]

    def host(shape, dtype):
        a = torch.empty(shape, dtype=dtype)
        return a.pin_memory() if pinned else a
    Xh = host(tuple(X.shape), X.dtype)
    Fh = host((w.T, w.d), X.dtype)
    Xh.copy_(X.cpu())
    Fh.copy_(t["F"].cpu())
    return dict(X=Xh, F=Fh, x_in=host((w.T, w.d), X.dtype), H=host((w.T, w.m), torch.float32),
                Y=host(tuple(X.shape), X.dtype))


def _call(w, t, hb, chunk, ws):
    s = w.scalars()
    mhc.mhc_forward_host(hb["X"], hb["F"], t["phi"], t["b_pre"], t["b_post"], t["b_res"],
                         s["alpha_pre"], s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"],
                         hb["x_in"], hb["H"], hb["Y"], ws, chunk_tokens=chunk)


def _workspace(chunk, w, dtype):
    return torch.empty(mhc.mhc_forward_host_workspace_bytes(chunk, w.n, w.d, dtype),
                       dtype=torch.uint8, device="cuda")


def _host_run(w, t, chunk, pinned=True):
    hb = _host_buffers(w, t, pinned)
    _call(w, t, hb, chunk, _workspace(chunk, w, t["X"].dtype))
    torch.cuda.synchronize()
    assert mhc.mhc_device_status() == 0
    return hb["x_in"], hb["H"], hb["Y"]


def _chunked_device(w, t, chunk):
    """mhc_pre + mhc_post called on each chunk of tokens, on the device."""
    s = w.scalars()
    X = t["X"]
    xs, Hs, Ys = [], [], []
    for t0 in range(0, w.T, chunk):
        Xc = X[t0:t0 + chunk].contiguous()
        Fc = t["F"][t0:t0 + chunk].contiguous()
        tc = Xc.shape[0]
        x_in = torch.empty(tc, w.d, dtype=X.dtype, device=X.device)
        H = torch.empty(tc, w.m, dtype=torch.float32, device=X.device)
        Y = torch.empty_like(Xc)
        mhc.mhc_pre(Xc, t["phi"], t["b_pre"], t["b_post"], t["b_res"], s["alpha_pre"], s["alpha_post"],
                    s["alpha_res"], s["eps"], s["t_max"], x_in, H)
        mhc.mhc_post(Xc, Fc, H, Y)
        xs.append(x_in)
        Hs.append(H)
        Ys.append(Y)
    torch.cuda.synchronize()
    return torch.cat(xs).cpu(), torch.cat(Hs).cpu(), torch.cat(Ys).cpu()


def _bits(a):
    return a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32)


# (T, n, d, dtype, chunk): the cluster path with a ragged last chunk, the two-pass path
# (n = 8), the generic path (fp32), one chunk larger than T, and chunks of one token
CASES = [
    (3000, 4, 1024, "bf16", 1024),
    (1500, 8, 512, "bf16", 512),
    (777, 2, 256, "f32", 200),
    (300, 4, 2048, "bf16", 4096),
    (5, 3, 512, "bf16", 1),
]


@pytest.mark.parametrize("T,n,d,dtype,chunk", CASES)
def test_forward_host_matches_device_chunks(T, n, d, dtype, chunk):
    w = wl.make_inputs(T=T, n=n, d=d, dtype=dtype, seed=11, outlier_frac=0.01)
    t = torch_inputs(w)
    host = _host_run(w, t, chunk)
    dev = _chunked_device(w, t, chunk)
    for name, a, b in zip(("x_in", "H", "X_out"), host, dev):
        assert torch.equal(_bits(a), _bits(b)), f"{name}: host path differs from the device path"


def test_forward_host_whole_batch_and_oracle():
    """T = 3000 in chunks of 1024 on the cluster path: equal to the one-call device result,
    and within the parity tolerance of the oracle on the first and the ragged last chunk."""
    w = wl.make_inputs(T=3000, n=4, d=1024, dtype="bf16", seed=12, outlier_frac=0.01)
    t = torch_inputs(w)
    if mhc.mhc_pre_path_for(1024, 4, 1024, torch.bfloat16) != mhc.mhc_pre_path_for(3000, 4, 1024, torch.bfloat16):
        pytest.skip("the chunk and the whole batch take different kernel paths on this device")
    host = _host_run(w, t, 1024)
    whole = [a.cpu() for a in run_gpu(w, inputs=t)]
    for name, a, b in zip(("x_in", "H", "X_out"), host, whole):
        assert torch.equal(_bits(a), _bits(b)), f"{name}: chunked host path differs from one device call"
    for lo, hi in ((0, 1024), (2048, 3000)):
        sub = w.tokens(np.arange(lo, hi))
        check_against_oracle(sub, tuple(a[lo:hi] for a in host), run_oracle(sub), f"tokens {lo}:{hi}")


def test_forward_host_pageable_memory():
    """Pageable host buffers give the same results (the copies are then staged by the driver)."""
    w = wl.make_inputs(T=700, n=4, d=1024, dtype="bf16", seed=13)
    t = torch_inputs(w)
    a = _host_run(w, t, 256, pinned=True)
    b = _host_run(w, t, 256, pinned=False)
    for x, y in zip(a, b):
        assert torch.equal(_bits(x), _bits(y))


def test_forward_host_reuses_workspace_across_calls():
    """Two calls queued back to back on one stream and one workspace, with no synchronisation
    between them: each sees its own inputs."""
    w1 = wl.make_inputs(T=900, n=4, d=1024, dtype="bf16", seed=14)
    w2 = wl.make_inputs(T=900, n=4, d=1024, dtype="bf16", seed=15)
    t1, t2 = torch_inputs(w1), torch_inputs(w2)
    ws = _workspace(128, w1, torch.bfloat16)
    hb1, hb2 = _host_buffers(w1, t1), _host_buffers(w2, t2)
    _call(w1, t1, hb1, 128, ws)
    _call(w2, t2, hb2, 128, ws)
    torch.cuda.synchronize()
    d1 = _chunked_device(w1, t1, 128)
    d2 = _chunked_device(w2, t2, 128)
    r = (hb1["x_in"], hb1["H"], hb1["Y"], hb2["x_in"], hb2["H"], hb2["Y"])
    for x, y in zip(r, d1 + d2):
        assert torch.equal(_bits(x), _bits(y))


def test_forward_host_two_host_threads():
    """Two host threads call mhc_forward_host at once, each on its own stream and workspace:
    the library's copy streams are shared, and each call still sees its own inputs."""
    import threading
    ws_ = [wl.make_inputs(T=700, n=4, d=1024, dtype="bf16", seed=16 + k) for k in range(2)]
    ts = [torch_inputs(w) for w in ws_]
    hbs = [_host_buffers(w, t) for w, t in zip(ws_, ts)]
    wss = [_workspace(256, w, torch.bfloat16) for w in ws_]
    streams = [torch.cuda.Stream() for _ in range(2)]
    errors = []

    def worker(k):
        try:
            with torch.cuda.stream(streams[k]):
                for _ in range(3):
                    _call(ws_[k], ts[k], hbs[k], 256, wss[k])
            streams[k].synchronize()
        except Exception as e:          # surfaced below
            errors.append(e)
    th = [threading.Thread(target=worker, args=(k,)) for k in range(2)]
    for t_ in th:
        t_.start()
    for t_ in th:
        t_.join()
    assert not errors, errors
    torch.cuda.synchronize()
    for k in range(2):
        ref = _chunked_device(ws_[k], ts[k], 256)
        for x, y in zip((hbs[k]["x_in"], hbs[k]["H"], hbs[k]["Y"]), ref):
            assert torch.equal(_bits(x), _bits(y))
