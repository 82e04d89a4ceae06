"""ctypes binding of ``libxlstm_mlstm.so``: argument marshalling only.

The names mirror the C ABI in ``include/xlstm_mlstm.h``.  ``load()`` binds the
library and raises if it is missing: there is no fallback path.  The
convenience wrappers ``mlstm_fwd`` / ``mlstm_step`` take torch CUDA tensors,
allocate outputs and workspace with torch (device memory is PyTorch's job
here), pass raw pointers and the current CUDA stream, and turn a non-OK status
into ``XlstmError``.  Every step of the computation runs in the library's
kernels.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libxlstm_mlstm.so")

OK, ERR_NULL, ERR_SHAPE, ERR_DTYPE, ERR_CHUNK, ERR_ALIGN, ERR_CUDA, ERR_TIMEOUT, \
    ERR_WORKSPACE, ERR_UNSUPPORTED = range(10)
F32, BF16 = 0, 1
FGATE_SIGMOID, FGATE_EXP = 0, 1
OGATE_SILU, OGATE_SIGMOID = 0, 1
PATH_AUTO, PATH_SIMT, PATH_TENSOR, PATH_TENSOR_TMEM, PATH_TENSOR_RS = 0, 1, 2, 3, 4

EXPORTED = ("xlstm_abi_version", "xlstm_status_string", "xlstm_mlstm_fwd_workspace_size",
            "xlstm_mlstm_fwd_workspace_size_ex", "xlstm_mlstm_fwd", "xlstm_mlstm_fwd_ex",
            "xlstm_mlstm_step", "xlstm_device_status", "xlstm_profile_begin", "xlstm_profile_end",
            "xlstm_mlstm_fwd_noalloc", "xlstm_selftest_wait_timeout", "xlstm_mlstm_headnorm_gate",
            "xlstm_mlstm_bwd_workspace_size", "xlstm_mlstm_bwd", "xlstm_slstm_fwd",
            "xlstm_mlstm_fwd_path", "xlstm_mlstm_seg_state_floats",
            "xlstm_mlstm_seg_state_workspace_size", "xlstm_mlstm_seg_state",
            "xlstm_mlstm_state_combine")
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class XlstmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class FwdOptions(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("segments", ctypes.c_int)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int),
                ("total_ms", ctypes.c_double)]


_lock = threading.Lock()
_lib = None


def load(path: str = LIB_PATH):
    """Load and bind the library.  Raises OSError if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise OSError(f"{path} is missing: build it with `python -m linear_rnn_mlstm_b200.build`"
                          " (the mLSTM ops have no other implementation)")
        lib = ctypes.CDLL(path)
        vp, fp, i, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.xlstm_abi_version.restype = i
        lib.xlstm_status_string.argtypes = [i]
        lib.xlstm_status_string.restype = ctypes.c_char_p
        lib.xlstm_mlstm_fwd_workspace_size.argtypes = [i] * 6 + [ctypes.POINTER(sz)]
        lib.xlstm_mlstm_fwd_workspace_size.restype = i
        lib.xlstm_mlstm_fwd_workspace_size_ex.argtypes = [i] * 6 + [ctypes.POINTER(FwdOptions),
                                                                   ctypes.POINTER(sz)]
        lib.xlstm_mlstm_fwd_workspace_size_ex.restype = i
        lib.xlstm_mlstm_fwd_path.argtypes = [i] * 3 + [ctypes.POINTER(FwdOptions), ctypes.POINTER(i)]
        lib.xlstm_mlstm_fwd_path.restype = i
        fwd_args = [vp] * 3 + [fp] * 3 + [vp] + [fp] * 6 + [i] * 7 + [vp, sz]
        lib.xlstm_mlstm_fwd.argtypes = fwd_args + [vp]
        lib.xlstm_mlstm_fwd.restype = i
        lib.xlstm_mlstm_fwd_ex.argtypes = fwd_args + [ctypes.POINTER(FwdOptions), vp]
        lib.xlstm_mlstm_fwd_ex.restype = i
        lib.xlstm_mlstm_step.argtypes = [vp] * 3 + [fp] * 3 + [vp] + [fp] * 3 + [i] * 5 + [vp]
        lib.xlstm_mlstm_step.restype = i
        lib.xlstm_device_status.argtypes = [vp]
        lib.xlstm_device_status.restype = i
        lib.xlstm_selftest_wait_timeout.argtypes = [i, vp]
        lib.xlstm_selftest_wait_timeout.restype = i
        lib.xlstm_mlstm_fwd_noalloc.argtypes = [vp] * 3 + [fp] * 3 + [vp] + [fp] * 6 + [i] * 7 + [vp]
        lib.xlstm_mlstm_fwd_noalloc.restype = i
        lib.xlstm_mlstm_headnorm_gate.argtypes = [vp] + [fp] * 3 + [vp] * 3 + [i] * 4 + \
            [ctypes.c_float, i, i, vp]
        lib.xlstm_mlstm_headnorm_gate.restype = i
        lib.xlstm_mlstm_bwd_workspace_size.argtypes = [i] * 6 + [ctypes.POINTER(sz)]
        lib.xlstm_mlstm_bwd_workspace_size.restype = i
        lib.xlstm_mlstm_bwd.argtypes = [vp] * 3 + [fp] * 3 + [vp] + [fp] * 2 + [vp] * 3 + \
            [fp] * 3 + [i] * 7 + [vp, sz, vp]
        lib.xlstm_mlstm_bwd.restype = i
        lib.xlstm_slstm_fwd.argtypes = [fp] * 14 + [i] * 5 + [vp]
        lib.xlstm_slstm_fwd.restype = i
        lib.xlstm_mlstm_seg_state_floats.argtypes = [i] * 3 + [ctypes.POINTER(sz)]
        lib.xlstm_mlstm_seg_state_floats.restype = i
        lib.xlstm_mlstm_seg_state_workspace_size.argtypes = [i] * 6 + [ctypes.POINTER(sz)]
        lib.xlstm_mlstm_seg_state_workspace_size.restype = i
        lib.xlstm_mlstm_seg_state.argtypes = [vp] * 2 + [fp] * 3 + [i] * 7 + [vp, sz, vp]
        lib.xlstm_mlstm_seg_state.restype = i
        lib.xlstm_mlstm_state_combine.argtypes = [fp, i] + [fp] * 6 + [i] * 3 + [vp]
        lib.xlstm_mlstm_state_combine.restype = i
        lib.xlstm_profile_begin.restype = i
        lib.xlstm_profile_end.argtypes = [ctypes.POINTER(KernelTime), i, ctypes.POINTER(i)]
        lib.xlstm_profile_end.restype = i
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().xlstm_status_string(int(status)).decode()


# ----------------------------------------------------- raw C entry points
def xlstm_abi_version() -> int:
    return load().xlstm_abi_version()


def xlstm_mlstm_fwd_workspace_size(B, NH, S, DH, chunk, dt, path=PATH_AUTO, segments=0):
    n = ctypes.c_size_t(0)
    opts = FwdOptions(path, segments)
    st = load().xlstm_mlstm_fwd_workspace_size_ex(B, NH, S, DH, chunk, dt, ctypes.byref(opts),
                                                   ctypes.byref(n))
    return st, n.value


def xlstm_mlstm_fwd_path(DH, chunk, dt, path=PATH_AUTO, segments=0):
    """(status, kernel family) the forward would run: PATH_SIMT or PATH_TENSOR."""
    out = ctypes.c_int(0)
    opts = FwdOptions(path, segments)
    st = load().xlstm_mlstm_fwd_path(DH, chunk, dt, ctypes.byref(opts), ctypes.byref(out))
    return st, out.value


def xlstm_mlstm_fwd(q, k, v, i_pre, f_pre, o_pre, h, C0, n0, m0, C_out, n_out, m_out,
                    B, NH, S, DH, chunk, dt, fg, workspace, workspace_bytes, stream,
                    path=PATH_AUTO, segments=0):
    """Pointers are ints (device addresses) or None; returns the status."""
    opts = FwdOptions(path, segments)
    return load().xlstm_mlstm_fwd_ex(q, k, v, i_pre, f_pre, o_pre, h, C0, n0, m0,
                                     C_out, n_out, m_out, B, NH, S, DH, chunk, dt, fg,
                                     workspace, workspace_bytes, ctypes.byref(opts), stream)


def xlstm_mlstm_fwd_noalloc(q, k, v, i_pre, f_pre, o_pre, h, C0, n0, m0, C_out, n_out, m_out,
                            B, NH, S, DH, chunk, dt, fg, stream):
    """The forward with the library's built-in scratch (no workspace argument)."""
    return load().xlstm_mlstm_fwd_noalloc(q, k, v, i_pre, f_pre, o_pre, h, C0, n0, m0,
                                          C_out, n_out, m_out, B, NH, S, DH, chunk, dt, fg, stream)


def xlstm_mlstm_step(q, k, v, i_pre, f_pre, o_pre, h, C, n, m, B, NH, DH, dt, fg, stream):
    return load().xlstm_mlstm_step(q, k, v, i_pre, f_pre, o_pre, h, C, n, m, B, NH, DH, dt, fg,
                                   stream)


def xlstm_mlstm_headnorm_gate(h, gamma, beta, skip_w, x_skip, z, y, B, NH, S, DH, eps, dt, og,
                              stream):
    return load().xlstm_mlstm_headnorm_gate(h, gamma, beta, skip_w, x_skip, z, y, B, NH, S, DH,
                                            float(eps), dt, og, stream)


def xlstm_mlstm_bwd_workspace_size(B, NH, S, DH, chunk, dt):
    n = ctypes.c_size_t(0)
    st = load().xlstm_mlstm_bwd_workspace_size(B, NH, S, DH, chunk, dt, ctypes.byref(n))
    return st, n.value


def xlstm_mlstm_bwd(q, k, v, i_pre, f_pre, o_pre, dh, dC, dn, dq, dk, dv, di, df, d_o,
                    B, NH, S, DH, chunk, dt, fg, workspace, workspace_bytes, stream):
    return load().xlstm_mlstm_bwd(q, k, v, i_pre, f_pre, o_pre, dh, dC, dn, dq, dk, dv, di, df,
                                  d_o, B, NH, S, DH, chunk, dt, fg, workspace, workspace_bytes,
                                  stream)


def xlstm_slstm_fwd(zx, ix, fx, ox, R, h, c0, n0, m0, h0, c_out, n_out, m_out, h_out,
                    B, NH, S, DH, fg, stream):
    return load().xlstm_slstm_fwd(zx, ix, fx, ox, R, h, c0, n0, m0, h0, c_out, n_out, m_out,
                                  h_out, B, NH, S, DH, fg, stream)


def xlstm_mlstm_seg_state_floats(B, NH, DH):
    n = ctypes.c_size_t(0)
    st = load().xlstm_mlstm_seg_state_floats(B, NH, DH, ctypes.byref(n))
    return st, n.value


def xlstm_mlstm_seg_state_workspace_size(B, NH, S, DH, chunk, dt):
    n = ctypes.c_size_t(0)
    st = load().xlstm_mlstm_seg_state_workspace_size(B, NH, S, DH, chunk, dt, ctypes.byref(n))
    return st, n.value


def xlstm_mlstm_seg_state(k, v, i_pre, f_pre, packed, B, NH, S, DH, chunk, dt, fg, workspace,
                          workspace_bytes, stream):
    return load().xlstm_mlstm_seg_state(k, v, i_pre, f_pre, packed, B, NH, S, DH, chunk, dt, fg,
                                        workspace, workspace_bytes, stream)


def xlstm_mlstm_state_combine(parts, count, C0, n0, m0, C_out, n_out, m_out, B, NH, DH, stream):
    return load().xlstm_mlstm_state_combine(parts, count, C0, n0, m0, C_out, n_out, m_out, B, NH,
                                            DH, stream)


def xlstm_device_status(stream) -> int:
    return load().xlstm_device_status(stream)


def xlstm_selftest_wait_timeout(limit_us: int, stream) -> int:
    return load().xlstm_selftest_wait_timeout(limit_us, stream)


def xlstm_profile_begin() -> int:
    return load().xlstm_profile_begin()


def xlstm_profile_end(max_kernels: int = 32):
    """Returns (status, {kernel name: (launches, total_ms)})."""
    arr = (KernelTime * max_kernels)()
    count = ctypes.c_int(0)
    st = load().xlstm_profile_end(arr, max_kernels, ctypes.byref(count))
    out = {}
    for i in range(min(count.value, max_kernels)):
        out[arr[i].name.decode()] = (arr[i].launches, arr[i].total_ms)
    return st, out


# ------------------------------------------------------ torch conveniences
def _torch():
    import torch
    return torch


def _dt(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check(t, name, shape, dtype, device):
    if t is None:
        return
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")


def _stream(device):
    return _torch().cuda.current_stream(device).cuda_stream


def mlstm_fwd(q, k, v, i_pre, f_pre, o_pre, chunk=64, fgate="sigmoid", C0=None, n0=None,
              m0=None, h=None, state_out=True, path=PATH_AUTO, segments=0, workspace=None):
    """Chunkwise forward.  Returns (h, C, n, m) (state None unless state_out)."""
    torch = _torch()
    B, NH, S, DH = q.shape
    dev = q.device
    dtype = q.dtype
    dt = _dt(q)
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, nm, (B, NH, S, DH), dtype, dev)
    _check(i_pre, "i_pre", (B, NH, S), torch.float32, dev)
    _check(f_pre, "f_pre", (B, NH, S), torch.float32, dev)
    _check(o_pre, "o_pre", (B, NH, S, DH), torch.float32, dev)
    _check(C0, "C0", (B, NH, DH, DH), torch.float32, dev)
    _check(n0, "n0", (B, NH, DH), torch.float32, dev)
    _check(m0, "m0", (B, NH), torch.float32, dev)
    if h is None:
        h = torch.empty((B, NH, S, DH), dtype=dtype, device=dev)
    _check(h, "h", (B, NH, S, DH), dtype, dev)
    C = n = m = None
    if state_out:
        C = torch.empty((B, NH, DH, DH), dtype=torch.float32, device=dev)
        n = torch.empty((B, NH, DH), dtype=torch.float32, device=dev)
        m = torch.empty((B, NH), dtype=torch.float32, device=dev)
    fg = FGATE_EXP if fgate == "exp" else FGATE_SIGMOID
    st, nbytes = xlstm_mlstm_fwd_workspace_size(B, NH, S, DH, chunk, dt, path, segments)
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_fwd_workspace_size")
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    st = xlstm_mlstm_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(i_pre), _ptr(f_pre), _ptr(o_pre),
                         _ptr(h), _ptr(C0), _ptr(n0), _ptr(m0), _ptr(C), _ptr(n), _ptr(m),
                         B, NH, S, DH, chunk, dt, fg, workspace.data_ptr(), workspace.numel(),
                         _stream(dev), path, segments)
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_fwd")
    return h, C, n, m


def seg_state_floats(B, NH, DH) -> int:
    st, n = xlstm_mlstm_seg_state_floats(B, NH, DH)
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_seg_state_floats")
    return n


def unpack_seg_state(packed, B, NH, DH):
    """Views (C', n', mloc, F) of one packed slice summary (layout of the C header)."""
    BH = B * NH
    o1 = BH * DH * DH
    o2 = o1 + BH * DH
    return (packed[:o1].view(B, NH, DH, DH), packed[o1:o2].view(B, NH, DH),
            packed[o2:o2 + BH].view(B, NH), packed[o2 + BH:o2 + 2 * BH].view(B, NH))


def mlstm_seg_state(k, v, i_pre, f_pre, chunk=64, fgate="sigmoid", packed=None, workspace=None):
    """Summary of one slice of a sequence (zero start): a flat float32 tensor of
    ``seg_state_floats`` floats, see ``unpack_seg_state``."""
    torch = _torch()
    B, NH, S, DH = k.shape
    dev, dtype, dt = k.device, k.dtype, _dt(k)
    _check(k, "k", (B, NH, S, DH), dtype, dev)
    _check(v, "v", (B, NH, S, DH), dtype, dev)
    _check(i_pre, "i_pre", (B, NH, S), torch.float32, dev)
    _check(f_pre, "f_pre", (B, NH, S), torch.float32, dev)
    nf = seg_state_floats(B, NH, DH)
    if packed is None:
        packed = torch.empty(nf, dtype=torch.float32, device=dev)
    _check(packed, "packed", (nf,), torch.float32, dev)
    st, nbytes = xlstm_mlstm_seg_state_workspace_size(B, NH, S, DH, chunk, dt)
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_seg_state_workspace_size")
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    fg = FGATE_EXP if fgate == "exp" else FGATE_SIGMOID
    st = xlstm_mlstm_seg_state(_ptr(k), _ptr(v), _ptr(i_pre), _ptr(f_pre), _ptr(packed), B, NH, S,
                               DH, chunk, dt, fg, workspace.data_ptr(), workspace.numel(),
                               _stream(dev))
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_seg_state")
    return packed


def mlstm_state_combine(parts, count, B, NH, DH, C0=None, n0=None, m0=None, out=None):
    """Fold the first ``count`` packed summaries of ``parts`` ([>= count, floats])
    onto (C0, n0, m0).  Returns (C', n', m)."""
    torch = _torch()
    dev = parts.device
    nf = seg_state_floats(B, NH, DH)
    if parts.dim() != 2 or parts.shape[1] != nf or parts.shape[0] < count:
        raise ValueError(f"parts must be [>= {count}, {nf}], got {tuple(parts.shape)}")
    _check(parts, "parts", tuple(parts.shape), torch.float32, dev)
    _check(C0, "C0", (B, NH, DH, DH), torch.float32, dev)
    _check(n0, "n0", (B, NH, DH), torch.float32, dev)
    _check(m0, "m0", (B, NH), torch.float32, dev)
    if out is None:
        out = (torch.empty((B, NH, DH, DH), dtype=torch.float32, device=dev),
               torch.empty((B, NH, DH), dtype=torch.float32, device=dev),
               torch.empty((B, NH), dtype=torch.float32, device=dev))
    C, n, m = out
    st = xlstm_mlstm_state_combine(_ptr(parts), count, _ptr(C0), _ptr(n0), _ptr(m0), _ptr(C),
                                   _ptr(n), _ptr(m), B, NH, DH, _stream(dev))
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_state_combine")
    return C, n, m


def mlstm_step(q, k, v, i_pre, f_pre, o_pre, C, n, m, fgate="sigmoid", h=None):
    """One decode token; (C, n, m) are updated in place.  Returns h."""
    torch = _torch()
    B, NH, DH = q.shape
    dev, dtype, dt = q.device, q.dtype, _dt(q)
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, nm, (B, NH, DH), dtype, dev)
    _check(i_pre, "i_pre", (B, NH), torch.float32, dev)
    _check(f_pre, "f_pre", (B, NH), torch.float32, dev)
    _check(o_pre, "o_pre", (B, NH, DH), torch.float32, dev)
    _check(C, "C", (B, NH, DH, DH), torch.float32, dev)
    _check(n, "n", (B, NH, DH), torch.float32, dev)
    _check(m, "m", (B, NH), torch.float32, dev)
    if h is None:
        h = torch.empty((B, NH, DH), dtype=dtype, device=dev)
    fg = FGATE_EXP if fgate == "exp" else FGATE_SIGMOID
    st = xlstm_mlstm_step(_ptr(q), _ptr(k), _ptr(v), _ptr(i_pre), _ptr(f_pre), _ptr(o_pre),
                          _ptr(h), _ptr(C), _ptr(n), _ptr(m), B, NH, DH, dt, fg, _stream(dev))
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_step")
    return h


def mlstm_headnorm_gate(h, gamma, beta, z, skip_w=None, x_skip=None, eps=1e-5, ogate="silu",
                        y=None):
    """Block epilogue after the cell: per-head GroupNorm of h [B, NH, S, DH],
    plus skip_w * x_skip, gated by act(z); x_skip, z and the returned y are
    [B, S, NH * DH].  Returns y."""
    torch = _torch()
    B, NH, S, DH = h.shape
    dev, dtype, dt = h.device, h.dtype, _dt(h)
    _check(h, "h", (B, NH, S, DH), dtype, dev)
    for t, nm in ((gamma, "gamma"), (beta, "beta"), (skip_w, "skip_w")):
        _check(t, nm, (NH * DH,), torch.float32, dev)
    _check(x_skip, "x_skip", (B, S, NH * DH), dtype, dev)
    _check(z, "z", (B, S, NH * DH), dtype, dev)
    if y is None:
        y = torch.empty((B, S, NH * DH), dtype=dtype, device=dev)
    _check(y, "y", (B, S, NH * DH), dtype, dev)
    if ogate not in ("silu", "sigmoid"):
        raise ValueError("ogate must be 'silu' or 'sigmoid'")
    og = OGATE_SILU if ogate == "silu" else OGATE_SIGMOID
    st = xlstm_mlstm_headnorm_gate(_ptr(h), _ptr(gamma), _ptr(beta), _ptr(skip_w), _ptr(x_skip),
                                   _ptr(z), _ptr(y), B, NH, S, DH, eps, dt, og, _stream(dev))
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_headnorm_gate")
    return y


def mlstm_bwd(q, k, v, i_pre, f_pre, o_pre, dh, dC=None, dn=None, chunk=64, fgate="sigmoid"):
    """Gradients of sum(dh h) + sum(dC C'_T) + sum(dn n'_T) through the forward
    from a zero state.  Returns dict dq, dk, dv (q's dtype), di, df, do (fp32)."""
    torch = _torch()
    B, NH, S, DH = q.shape
    dev, dtype, dt = q.device, q.dtype, _dt(q)
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (dh, "dh")):
        _check(t, nm, (B, NH, S, DH), dtype, dev)
    _check(i_pre, "i_pre", (B, NH, S), torch.float32, dev)
    _check(f_pre, "f_pre", (B, NH, S), torch.float32, dev)
    _check(o_pre, "o_pre", (B, NH, S, DH), torch.float32, dev)
    _check(dC, "dC", (B, NH, DH, DH), torch.float32, dev)
    _check(dn, "dn", (B, NH, DH), torch.float32, dev)
    out = {nm: torch.empty((B, NH, S, DH), dtype=dtype, device=dev) for nm in ("dq", "dk", "dv")}
    out["di"] = torch.empty((B, NH, S), dtype=torch.float32, device=dev)
    out["df"] = torch.empty((B, NH, S), dtype=torch.float32, device=dev)
    out["do"] = torch.empty((B, NH, S, DH), dtype=torch.float32, device=dev)
    st, nbytes = xlstm_mlstm_bwd_workspace_size(B, NH, S, DH, chunk, dt)
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_bwd_workspace_size")
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    fg = FGATE_EXP if fgate == "exp" else FGATE_SIGMOID
    st = xlstm_mlstm_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(i_pre), _ptr(f_pre), _ptr(o_pre),
                         _ptr(dh), _ptr(dC), _ptr(dn), _ptr(out["dq"]), _ptr(out["dk"]),
                         _ptr(out["dv"]), _ptr(out["di"]), _ptr(out["df"]), _ptr(out["do"]),
                         B, NH, S, DH, chunk, dt, fg, ws.data_ptr(), ws.numel(), _stream(dev))
    if st != OK:
        raise XlstmError(st, "xlstm_mlstm_bwd")
    return out


def slstm_fwd(zx, ix, fx, ox, R, fgate="sigmoid", c0=None, n0=None, m0=None, h0=None):
    """sLSTM forward on fp32 CUDA tensors zx, ix, fx, ox [B, NH, S, DH] and
    R [NH, 4, DH, DH].  Returns (h, c, n, m, h_last)."""
    torch = _torch()
    B, NH, S, DH = zx.shape
    dev = zx.device
    for t, nm in ((zx, "zx"), (ix, "ix"), (fx, "fx"), (ox, "ox")):
        _check(t, nm, (B, NH, S, DH), torch.float32, dev)
    _check(R, "R", (NH, 4, DH, DH), torch.float32, dev)
    for t, nm in ((c0, "c0"), (n0, "n0"), (m0, "m0"), (h0, "h0")):
        _check(t, nm, (B, NH, DH), torch.float32, dev)
    h = torch.empty((B, NH, S, DH), dtype=torch.float32, device=dev)
    st_out = [torch.empty((B, NH, DH), dtype=torch.float32, device=dev) for _ in range(4)]
    fg = FGATE_EXP if fgate == "exp" else FGATE_SIGMOID
    st = xlstm_slstm_fwd(_ptr(zx), _ptr(ix), _ptr(fx), _ptr(ox), _ptr(R), _ptr(h), _ptr(c0),
                         _ptr(n0), _ptr(m0), _ptr(h0), *(_ptr(t) for t in st_out),
                         B, NH, S, DH, fg, _stream(dev))
    if st != OK:
        raise XlstmError(st, "xlstm_slstm_fwd")
    return (h, *st_out)
