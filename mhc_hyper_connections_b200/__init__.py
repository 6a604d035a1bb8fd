"""mhc_hyper_connections_b200 -- B200-native (sm_100a) mHC layer: pre and post stages, their
backward, and the Amax gain diagnostic.

Thin Python binding over the C ABI in include/mhc.h (libmhc_b200.so, built in-tree by
``python -m mhc_hyper_connections_b200.build``).  The functions here only marshal
arguments: every step of the path runs in the library's CUDA kernels, and there is no
CPU fallback -- if the library is missing the calls raise.

    mhc_pre(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, eps, t_max,
            x_in, H)                -> writes x_in [T, d] and H [T, n*n+2n]
    mhc_pre_hc(..., eps, x_in, H)   -> the same with the HC comparison maps (bias + alpha tanh)
    mhc_post(X, F_out, H, X_out)    -> writes X_out [T, n, d]
    mhc_pre_train(..., x_in, H, h)  -> mhc_pre plus the normalised projection h [T, m]
    mhc_backward(X, F_out, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res,
                 eps, t_max, H, h, dX_out, dx_in, dX, dF_out, dphi, db_pre, db_post,
                 db_res, dalpha, workspace)  -> the gradients of <dX_out, X'> + <dx_in, x_in>
    mhc_backward_noalloc(...)       -> the same, in the library's fixed scratch array
    mhc_amax_gain(H_layers, gain)   -> per-prefix row / column gains of H_res(l) ... H_res(1)

Tensors are torch CUDA tensors (contiguous; X/F_out/x_in/X_out bf16 or fp32, phi, biases
and H fp32).  Calls are asynchronous on the current torch stream unless ``stream`` (a
torch.cuda.Stream or a raw cudaStream_t integer) is given.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = ["mhc_pre", "mhc_pre_with_path", "mhc_pre_hc", "mhc_pre_train", "mhc_post",
           "mhc_forward_host", "mhc_forward_host_workspace_bytes", "mhc_backward",
           "mhc_backward_workspace_bytes", "mhc_backward_noalloc", "NOALLOC_SCRATCH_BYTES",
           "mhc_amax_gain", "mhc_pre_path_for", "mhc_pre_path_ok", "mhc_device_status",
           "mhc_debug_pre_stop_after", "mhc_debug_backward_stop_after",
           "MhcError",
           "MHC_F32", "MHC_BF16", "PRE_AUTO", "PRE_GENERIC", "PRE_CLUSTER_TC", "PRE_TWO_PASS_TC", "library_path",
           "load_library", "EXPORTED_SYMBOLS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmhc_b200.so")

MHC_F32, MHC_BF16 = 0, 1
NOALLOC_SCRATCH_BYTES = 32 << 20      # the fixed scratch array of mhc_backward_noalloc
PRE_AUTO, PRE_GENERIC, PRE_CLUSTER_TC, PRE_TWO_PASS_TC = 0, 1, 2, 3
_STATUS = {0: "MHC_OK", 1: "MHC_ERR_NULL", 2: "MHC_ERR_SHAPE", 3: "MHC_ERR_ALIGN",
           4: "MHC_ERR_DTYPE", 5: "MHC_ERR_UNSUPPORTED", 6: "MHC_ERR_CUDA", 7: "MHC_ERR_ALIAS",
           8: "MHC_ERR_WORKSPACE"}

# Every function include/mhc.h declares.
EXPORTED_SYMBOLS = ("mhc_pre", "mhc_pre_with_path", "mhc_pre_hc", "mhc_pre_train", "mhc_pre_path_for",
                    "mhc_pre_path_ok", "mhc_post", "mhc_forward_host_workspace_bytes", "mhc_forward_host",
                    "mhc_backward_workspace_bytes", "mhc_backward", "mhc_backward_noalloc",
                    "mhc_amax_gain", "mhc_status_string",
                    "mhc_last_error", "mhc_device_status", "mhc_debug_pre_stop_after",
                    "mhc_debug_backward_stop_after")

_lock = threading.Lock()
_lib = None


class MhcError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        self.name = _STATUS.get(status, str(status))
        super().__init__(f"{where}: {self.name}" + (f" ({detail})" if detail else ""))


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libmhc_b200.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"CUDA library {_LIB_PATH} is missing: build it with "
                               "`python -m mhc_hyper_connections_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, fp, i64, ci, cf = (ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                               ctypes.c_float)
        pre_args = [vp, fp, fp, fp, fp, cf, cf, cf, i64, ci, ci, cf, ci, ci, vp, fp, vp]
        lib.mhc_pre.argtypes = pre_args
        lib.mhc_pre.restype = ci
        lib.mhc_pre_with_path.argtypes = pre_args + [ci]
        lib.mhc_pre_with_path.restype = ci
        lib.mhc_pre_hc.argtypes = pre_args[:12] + pre_args[13:] + [ci]
        lib.mhc_pre_hc.restype = ci
        lib.mhc_pre_train.argtypes = pre_args[:-1] + [fp, vp]
        lib.mhc_pre_train.restype = ci
        lib.mhc_backward_workspace_bytes.argtypes = [i64, ci, ci]
        lib.mhc_backward_workspace_bytes.restype = ctypes.c_size_t
        lib.mhc_backward.argtypes = ([vp, vp, fp, fp, fp, fp, cf, cf, cf, fp, fp, i64, ci, ci, cf, ci, ci,
                                      vp, vp, vp, vp, fp, fp, fp, fp, fp, vp, ctypes.c_size_t, vp])
        lib.mhc_backward.restype = ci
        lib.mhc_backward_noalloc.argtypes = lib.mhc_backward.argtypes[:-3] + [vp]
        lib.mhc_backward_noalloc.restype = ci
        lib.mhc_amax_gain.argtypes = [fp, ci, i64, ci, fp, vp]
        lib.mhc_amax_gain.restype = ci
        lib.mhc_pre_path_for.argtypes = [i64, ci, ci, ci]
        lib.mhc_pre_path_for.restype = ci
        lib.mhc_pre_path_ok.argtypes = [i64, ci, ci, ci, ci]
        lib.mhc_pre_path_ok.restype = ci
        lib.mhc_post.argtypes = [vp, vp, fp, i64, ci, ci, ci, vp, vp]
        lib.mhc_post.restype = ci
        lib.mhc_forward_host_workspace_bytes.argtypes = [i64, ci, ci, ci]
        lib.mhc_forward_host_workspace_bytes.restype = ctypes.c_size_t
        lib.mhc_forward_host.argtypes = ([vp, vp, fp, fp, fp, fp, cf, cf, cf, i64, ci, ci, cf, ci, ci,
                                          vp, fp, vp, i64, vp, ctypes.c_size_t, vp])
        lib.mhc_forward_host.restype = ci
        lib.mhc_status_string.argtypes = [ci]
        lib.mhc_status_string.restype = ctypes.c_char_p
        lib.mhc_last_error.argtypes = []
        lib.mhc_last_error.restype = ctypes.c_char_p
        lib.mhc_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
        lib.mhc_device_status.restype = ci
        lib.mhc_debug_pre_stop_after.argtypes = [ctypes.c_int32, ctypes.c_uint32]
        lib.mhc_debug_pre_stop_after.restype = ci
        lib.mhc_debug_backward_stop_after.argtypes = [ctypes.c_int32, ctypes.c_uint32]
        lib.mhc_debug_backward_stop_after.restype = ci
        _lib = lib
    return _lib


def _check(status: int, where: str):
    if status != 0:
        lib = load_library()
        detail = lib.mhc_status_string(status).decode()
        if status == 6:
            detail += "; " + lib.mhc_last_error().decode()
        raise MhcError(status, where, detail)


def _dt(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return MHC_BF16
    if t.dtype == torch.float32:
        return MHC_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t, name, dtype=None, device=None) -> int:
    import torch
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch tensor or raw device pointer")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor (the library takes device pointers)")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def _stream(stream, device) -> int:
    import torch
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def mhc_pre_with_path(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res,
                      eps, t_max, x_in, H, stream=None, path: int = PRE_AUTO):
    """Pre stage on an explicit kernel path (see mhc_pre)."""
    import torch
    T, n, d = X.shape
    dev = X.device
    f32 = torch.float32
    m = n * n + 2 * n
    if tuple(phi.shape) != (n * d, m) or tuple(x_in.shape) != (T, d) or tuple(H.shape) != (T, m):
        raise ValueError("mhc_pre: shapes must be phi [n*d, m], x_in [T, d], H [T, m]")
    if b_pre.numel() != n or b_post.numel() != n or b_res.numel() != n * n:
        raise ValueError("mhc_pre: b_pre/b_post need n entries, b_res n*n")
    ptrs = dict(X=_ptr(X, "X", device=dev), phi=_ptr(phi, "phi", f32, dev),
                b_pre=_ptr(b_pre, "b_pre", f32, dev), b_post=_ptr(b_post, "b_post", f32, dev),
                b_res=_ptr(b_res, "b_res", f32, dev), x_in=_ptr(x_in, "x_in", X.dtype, dev),
                H=_ptr(H, "H", f32, dev))
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.mhc_pre_with_path(ptrs["X"], ptrs["phi"], ptrs["b_pre"], ptrs["b_post"],
                                   ptrs["b_res"], float(alpha_pre), float(alpha_post),
                                   float(alpha_res), T, n, d, float(eps), int(t_max), _dt(X),
                                   ptrs["x_in"], ptrs["H"], _stream(stream, dev), int(path))
    _check(st, "mhc_pre")


def mhc_pre_hc(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, eps, x_in, H,
               stream=None, path: int = PRE_AUTO):
    """Pre stage with the HC comparison maps: H = b + alpha tanh(h) for every coefficient
    (no sigmoid, no Sinkhorn) and x_in = H_pre X; same shapes as mhc_pre."""
    import torch
    T, n, d = X.shape
    dev = X.device
    f32 = torch.float32
    m = n * n + 2 * n
    if tuple(phi.shape) != (n * d, m) or tuple(x_in.shape) != (T, d) or tuple(H.shape) != (T, m):
        raise ValueError("mhc_pre_hc: shapes must be phi [n*d, m], x_in [T, d], H [T, m]")
    if b_pre.numel() != n or b_post.numel() != n or b_res.numel() != n * n:
        raise ValueError("mhc_pre_hc: b_pre/b_post need n entries, b_res n*n")
    ptrs = dict(X=_ptr(X, "X", device=dev), phi=_ptr(phi, "phi", f32, dev),
                b_pre=_ptr(b_pre, "b_pre", f32, dev), b_post=_ptr(b_post, "b_post", f32, dev),
                b_res=_ptr(b_res, "b_res", f32, dev), x_in=_ptr(x_in, "x_in", X.dtype, dev),
                H=_ptr(H, "H", f32, dev))
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.mhc_pre_hc(ptrs["X"], ptrs["phi"], ptrs["b_pre"], ptrs["b_post"], ptrs["b_res"],
                            float(alpha_pre), float(alpha_post), float(alpha_res), T, n, d,
                            float(eps), _dt(X), ptrs["x_in"], ptrs["H"], _stream(stream, dev),
                            int(path))
    _check(st, "mhc_pre_hc")


def mhc_pre(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, eps, t_max,
            x_in, H, stream=None):
    """Pre stage: x_in = H_pre X and H = [H_pre | H_res | H_post] for every token.

    X [T, n, d] (bf16/fp32), phi [n*d, n*n+2n] fp32, b_pre/b_post [n], b_res [n, n] fp32;
    outputs x_in [T, d] (X's dtype) and H [T, n*n+2n] fp32, written in place."""
    mhc_pre_with_path(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, eps,
                      t_max, x_in, H, stream, PRE_AUTO)


def mhc_post(X, F_out, H, X_out, stream=None):
    """Post stage: X_out = H_res X + H_post^T F_out for every token (written in place)."""
    import torch
    T, n, d = X.shape
    dev = X.device
    if tuple(F_out.shape) != (T, d) or tuple(H.shape) != (T, n * n + 2 * n) or \
            tuple(X_out.shape) != (T, n, d):
        raise ValueError("mhc_post: shapes must be F_out [T, d], H [T, m], X_out [T, n, d]")
    px = _ptr(X, "X", device=dev)
    pf = _ptr(F_out, "F_out", X.dtype, dev)
    ph = _ptr(H, "H", torch.float32, dev)
    po = _ptr(X_out, "X_out", X.dtype, dev)
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.mhc_post(px, pf, ph, T, n, d, _dt(X), po, _stream(stream, dev))
    _check(st, "mhc_post")


def _host_ptr(t, name, dtype=None) -> int:
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch tensor in host memory")
    if t.is_cuda:
        raise ValueError(f"{name}: must be a host (CPU) tensor; pinned memory lets the copies overlap")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def mhc_forward_host_workspace_bytes(chunk_tokens: int, n: int, d: int, dtype) -> int:
    """Device workspace bytes mhc_forward_host needs for chunks of chunk_tokens tokens."""
    import torch
    dt = MHC_BF16 if dtype == torch.bfloat16 else MHC_F32 if dtype == torch.float32 else None
    if dt is None:
        raise TypeError(f"unsupported dtype {dtype}")
    v = load_library().mhc_forward_host_workspace_bytes(int(chunk_tokens), int(n), int(d), dt)
    if v == 0:
        raise MhcError(2, "mhc_forward_host_workspace_bytes", "chunk_tokens, n or d out of range")
    return v


def mhc_forward_host(X_h, F_out_h, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res,
                     eps, t_max, x_in_h, H_h, X_out_h, workspace, chunk_tokens: int = 1024,
                     stream=None):
    """mhc_pre then mhc_post on activations in host memory (X_h [T, n, d], F_out_h [T, d];
    outputs x_in_h [T, d], H_h [T, m], X_out_h [T, n, d], all CPU tensors, pinned for overlap).
    The parameters and the uint8 workspace (mhc_forward_host_workspace_bytes) are CUDA tensors.
    Asynchronous on `stream`: synchronise it before reading the outputs."""
    import torch
    T, n, d = X_h.shape
    m = n * n + 2 * n
    dev = phi.device
    f32 = torch.float32
    if tuple(F_out_h.shape) != (T, d) or tuple(x_in_h.shape) != (T, d) or tuple(H_h.shape) != (T, m) \
            or tuple(X_out_h.shape) != (T, n, d) or tuple(phi.shape) != (n * d, m):
        raise ValueError("mhc_forward_host: shapes must be F_out_h, x_in_h [T, d], H_h [T, m], "
                         "X_out_h [T, n, d], phi [n*d, m]")
    if b_pre.numel() != n or b_post.numel() != n or b_res.numel() != n * n:
        raise ValueError("mhc_forward_host: b_pre/b_post need n entries, b_res n*n")
    hp = dict(X=_host_ptr(X_h, "X_h"), F=_host_ptr(F_out_h, "F_out_h", X_h.dtype),
              xin=_host_ptr(x_in_h, "x_in_h", X_h.dtype), H=_host_ptr(H_h, "H_h", f32),
              Y=_host_ptr(X_out_h, "X_out_h", X_h.dtype))
    dp = dict(phi=_ptr(phi, "phi", f32, dev), b_pre=_ptr(b_pre, "b_pre", f32, dev),
              b_post=_ptr(b_post, "b_post", f32, dev), b_res=_ptr(b_res, "b_res", f32, dev),
              ws=_ptr(workspace, "workspace", torch.uint8, dev))
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.mhc_forward_host(hp["X"], hp["F"], dp["phi"], dp["b_pre"], dp["b_post"], dp["b_res"],
                                  float(alpha_pre), float(alpha_post), float(alpha_res), T, n, d,
                                  float(eps), int(t_max), _dt(X_h), hp["xin"], hp["H"], hp["Y"],
                                  int(chunk_tokens), dp["ws"], workspace.numel(), _stream(stream, dev))
    _check(st, "mhc_forward_host")


def mhc_pre_train(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, eps, t_max,
                  x_in, H, h, stream=None):
    """mhc_pre plus the normalised projection h [T, n*n+2n] fp32 that mhc_backward needs."""
    import torch
    T, n, d = X.shape
    dev = X.device
    f32 = torch.float32
    m = n * n + 2 * n
    if tuple(phi.shape) != (n * d, m) or tuple(x_in.shape) != (T, d) or tuple(H.shape) != (T, m) \
            or tuple(h.shape) != (T, m):
        raise ValueError("mhc_pre_train: shapes must be phi [n*d, m], x_in [T, d], H and h [T, m]")
    if b_pre.numel() != n or b_post.numel() != n or b_res.numel() != n * n:
        raise ValueError("mhc_pre_train: b_pre/b_post need n entries, b_res n*n")
    ptrs = dict(X=_ptr(X, "X", device=dev), phi=_ptr(phi, "phi", f32, dev),
                b_pre=_ptr(b_pre, "b_pre", f32, dev), b_post=_ptr(b_post, "b_post", f32, dev),
                b_res=_ptr(b_res, "b_res", f32, dev), x_in=_ptr(x_in, "x_in", X.dtype, dev),
                H=_ptr(H, "H", f32, dev), h=_ptr(h, "h", f32, dev))
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.mhc_pre_train(ptrs["X"], ptrs["phi"], ptrs["b_pre"], ptrs["b_post"], ptrs["b_res"],
                               float(alpha_pre), float(alpha_post), float(alpha_res), T, n, d,
                               float(eps), int(t_max), _dt(X), ptrs["x_in"], ptrs["H"], ptrs["h"],
                               _stream(stream, dev))
    _check(st, "mhc_pre_train")


def mhc_backward_workspace_bytes(T: int, n: int, d: int) -> int:
    """Bytes of device workspace mhc_backward needs (0 for a shape it rejects)."""
    return int(load_library().mhc_backward_workspace_bytes(int(T), int(n), int(d)))


def _backward_shapes(where, X, F_out, phi, b_pre, b_post, b_res, H, h, dX_out, dx_in, dX,
                     dF_out, dphi, db_pre, db_post, db_res, dalpha):
    """Check the shapes the backward reads and writes: the C ABI sees only pointers, so a
    tensor smaller than its shape here would be read or written past its end."""
    import torch
    if X.dim() != 3:
        raise ValueError(f"{where}: X must be [T, n, d]")
    T, n, d = X.shape
    m = n * n + 2 * n
    full = (("F_out", F_out, (T, d)), ("dx_in", dx_in, (T, d)), ("dF_out", dF_out, (T, d)),
            ("dX_out", dX_out, (T, n, d)), ("dX", dX, (T, n, d)), ("phi", phi, (n * d, m)),
            ("dphi", dphi, (n * d, m)), ("H", H, (T, m)), ("h", h, (T, m)))
    for name, t, shape in full:
        if isinstance(t, torch.Tensor) and tuple(t.shape) != shape:
            raise ValueError(f"{where}: {name} has shape {tuple(t.shape)}, expected {shape}")
    counts = (("b_pre", b_pre, n), ("b_post", b_post, n), ("b_res", b_res, n * n),
              ("db_pre", db_pre, n), ("db_post", db_post, n), ("db_res", db_res, n * n),
              ("dalpha", dalpha, 3))
    for name, t, cnt in counts:
        if isinstance(t, torch.Tensor) and t.numel() != cnt:
            raise ValueError(f"{where}: {name} needs {cnt} entries, has {t.numel()}")


def mhc_backward(X, F_out, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, eps, t_max,
                 H, h, dX_out, dx_in, dX, dF_out, dphi, db_pre, db_post, db_res, dalpha, workspace,
                 stream=None):
    """Gradients of <dX_out, X'> + <dx_in, x_in> (see include/mhc.h), written in place:
    dX [T,n,d], dF_out [T,d] in X's dtype; dphi [n*d, m], db_pre [n], db_post [n],
    db_res [n, n], dalpha [3] = (pre, post, res) fp32.  workspace: a CUDA tensor of at least
    mhc_backward_workspace_bytes(T, n, d) bytes."""
    import torch
    _backward_shapes("mhc_backward", X, F_out, phi, b_pre, b_post, b_res, H, h, dX_out, dx_in, dX,
                     dF_out, dphi, db_pre, db_post, db_res, dalpha)
    T, n, d = X.shape
    dev = X.device
    f32 = torch.float32
    dt = X.dtype
    p = {k: _ptr(v, k, dt, dev) for k, v in dict(X=X, F_out=F_out, dX_out=dX_out, dx_in=dx_in,
                                                  dX=dX, dF_out=dF_out).items()}
    q = {k: _ptr(v, k, f32, dev) for k, v in dict(phi=phi, b_pre=b_pre, b_post=b_post, b_res=b_res,
                                                   H=H, h=h, dphi=dphi, db_pre=db_pre,
                                                   db_post=db_post, db_res=db_res,
                                                   dalpha=dalpha).items()}
    ws = _ptr(workspace, "workspace", device=dev)
    nbytes = workspace.numel() * workspace.element_size()
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.mhc_backward(p["X"], p["F_out"], q["phi"], q["b_pre"], q["b_post"], q["b_res"],
                              float(alpha_pre), float(alpha_post), float(alpha_res), q["H"], q["h"],
                              T, n, d, float(eps), int(t_max), _dt(X), p["dX_out"], p["dx_in"],
                              p["dX"], p["dF_out"], q["dphi"], q["db_pre"], q["db_post"],
                              q["db_res"], q["dalpha"], ws, nbytes, _stream(stream, dev))
    _check(st, "mhc_backward")


def mhc_backward_noalloc(X, F_out, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res,
                         eps, t_max, H, h, dX_out, dx_in, dX, dF_out, dphi, db_pre, db_post,
                         db_res, dalpha, stream=None):
    """mhc_backward for callers that cannot allocate device memory: the same gradients, with
    the workspace in the library's fixed NOALLOC_SCRATCH_BYTES array instead of a caller
    buffer.  Raises MhcError(MHC_ERR_WORKSPACE) for sizes that need more.  All calls on a
    device share that array, so calls that overlap on the GPU must be ordered."""
    import torch
    _backward_shapes("mhc_backward_noalloc", X, F_out, phi, b_pre, b_post, b_res, H, h, dX_out,
                     dx_in, dX, dF_out, dphi, db_pre, db_post, db_res, dalpha)
    T, n, d = X.shape
    dev = X.device
    f32 = torch.float32
    dt = X.dtype
    p = {k: _ptr(v, k, dt, dev) for k, v in dict(X=X, F_out=F_out, dX_out=dX_out, dx_in=dx_in,
                                                  dX=dX, dF_out=dF_out).items()}
    q = {k: _ptr(v, k, f32, dev) for k, v in dict(phi=phi, b_pre=b_pre, b_post=b_post, b_res=b_res,
                                                   H=H, h=h, dphi=dphi, db_pre=db_pre,
                                                   db_post=db_post, db_res=db_res,
                                                   dalpha=dalpha).items()}
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.mhc_backward_noalloc(p["X"], p["F_out"], q["phi"], q["b_pre"], q["b_post"],
                                      q["b_res"], float(alpha_pre), float(alpha_post),
                                      float(alpha_res), q["H"], q["h"], T, n, d, float(eps),
                                      int(t_max), _dt(X), p["dX_out"], p["dx_in"], p["dX"],
                                      p["dF_out"], q["dphi"], q["db_pre"], q["db_post"],
                                      q["db_res"], q["dalpha"], _stream(stream, dev))
    _check(st, "mhc_backward_noalloc")


def mhc_amax_gain(H_layers, gain, stream=None):
    """Amax Gain Magnitude of composite residual maps: H_layers [L, T, n*n+2n] fp32 (each
    layer's H from mhc_pre, stacked) -> gain [L, T, 2] fp32 = (largest absolute row sum,
    largest absolute column sum) of H_res(l) ... H_res(1) for every prefix l."""
    import torch
    L, T, m = H_layers.shape
    n = int(round(((4 + 4 * m) ** 0.5 - 2) / 2))
    if n * n + 2 * n != m or tuple(gain.shape) != (L, T, 2):
        raise ValueError("mhc_amax_gain: H_layers [L, T, n*n+2n] and gain [L, T, 2]")
    dev = H_layers.device
    hp = _ptr(H_layers, "H_layers", torch.float32, dev)
    gp = _ptr(gain, "gain", torch.float32, dev)
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.mhc_amax_gain(hp, L, T, n, gp, _stream(stream, dev))
    _check(st, "mhc_amax_gain")


def mhc_device_status() -> int:
    """Read and clear the tensor-core kernel's device status word (0 = every bounded wait
    completed; otherwise bits naming the waits that expired)."""
    code = ctypes.c_uint32(0)
    _check(load_library().mhc_device_status(ctypes.byref(code)), "mhc_device_status")
    return int(code.value)


def mhc_debug_pre_stop_after(tiles: int, wait_limit_us: int = 1_000_000) -> None:
    """Test hook of the tensor-core pre kernel's failure path: later launches stop loading
    after `tiles` token tiles per cluster (tiles < 0 restores normal operation) and give up
    a wait after `wait_limit_us` microseconds.  The waits that depend on the tiles never
    loaded expire, the kernel returns early and mhc_device_status() reports it."""
    _check(load_library().mhc_debug_pre_stop_after(int(tiles), int(wait_limit_us)),
           "mhc_debug_pre_stop_after")


def mhc_debug_backward_stop_after(stages: int, wait_limit_us: int = 1_000_000) -> None:
    """Test hook of the backward's tensor-core dX / dphi step: later launches stop loading
    after `stages` 64-token stages per CTA (stages < 0 restores normal operation) and give up
    a wait after `wait_limit_us` microseconds; mhc_device_status() then reports bits 24-31."""
    _check(load_library().mhc_debug_backward_stop_after(int(stages), int(wait_limit_us)),
           "mhc_debug_backward_stop_after")


def mhc_pre_path_ok(T: int, n: int, d: int, dtype, path: int) -> bool:
    """Whether kernel path `path` can run this shape on the current device."""
    import torch
    dt = dtype if isinstance(dtype, int) else (MHC_BF16 if dtype == torch.bfloat16 else MHC_F32)
    return bool(load_library().mhc_pre_path_ok(int(T), int(n), int(d), dt, int(path)))


def mhc_pre_path_for(T: int, n: int, d: int, dtype) -> int:
    """Kernel path mhc_pre would take on the current device (PRE_GENERIC, PRE_CLUSTER_TC or
    PRE_TWO_PASS_TC)."""
    import torch
    dt = dtype if isinstance(dtype, int) else (MHC_BF16 if dtype == torch.bfloat16 else MHC_F32)
    return int(load_library().mhc_pre_path_for(int(T), int(n), int(d), dt))
