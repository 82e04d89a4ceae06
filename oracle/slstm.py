"""Python side of the float64 sLSTM oracle (``slstm_oracle.c``; test
infrastructure only).  "xLSTM: Extended Long Short-Term Memory" section 2.2:
scalar memory cells with exponential gating, a normaliser state, the
stabiliser m_t, and memory mixing through recurrent connections from h_{t-1}
to the cell input and the gates, within each head.

Shapes: zx, ix, fx, ox [B, NH, S, DH] (input-projection pre-activations of the
cell input z and the gates i, f, o, bias included); R [NH, 4, DH, DH] (gate
order z, i, f, o; row = receiving unit, column = unit of h_{t-1}); state c, n,
m, h [B, NH, DH].  Inputs may be numpy arrays or torch tensors; they are
converted exactly to float64.
"""
from __future__ import annotations

import ctypes
import threading

import numpy as np

from . import _SLSTM_LIB, _build_one, _SLSTM_SRC, _f64, _ptr

_lock = threading.Lock()
_lib = None


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    lib.slstm_oracle_fwd.argtypes = [dp] * 14 + [ctypes.c_long] * 4 + [ctypes.c_int] * 2
    lib.slstm_oracle_fwd.restype = ctypes.c_int
    return lib


def _load(path=None):
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(_build_one(_SLSTM_SRC, _SLSTM_LIB, False)))
    return _lib


def fwd(zx, ix, fx, ox, R, fgate="sigmoid", c0=None, n0=None, m0=None, h0=None, raw=False,
        lib_path=None):
    """Returns (h [B,NH,S,DH], c, n, m, h_last [B,NH,DH]) as float64 arrays; the
    final c, n are in stabilised units (raw units when ``raw``)."""
    zx = _f64(zx)
    if zx.ndim != 4:
        raise ValueError("zx must be [B, NH, S, DH]")
    B, NH, S, DH = zx.shape
    ix, fx, ox = (_f64(a, zx.shape) for a in (ix, fx, ox))
    R = _f64(R, (NH, 4, DH, DH))
    st = [_f64(a, (B, NH, DH)) for a in (c0, n0, m0, h0)]
    if fgate not in ("sigmoid", "exp"):
        raise ValueError("fgate must be 'sigmoid' or 'exp'")
    h = np.empty((B, NH, S, DH), np.float64)
    outs = [np.empty((B, NH, DH), np.float64) for _ in range(4)]
    rc = _load(lib_path).slstm_oracle_fwd(
        _ptr(zx), _ptr(ix), _ptr(fx), _ptr(ox), _ptr(R), _ptr(h), *(_ptr(a) for a in st),
        *(_ptr(a) for a in outs), B, NH, S, DH, 1 if fgate == "exp" else 0, 0 if raw else 1)
    if rc != 0:
        raise MemoryError("sLSTM oracle could not allocate its per-head state")
    return (h, *outs)
