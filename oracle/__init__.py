"""Float64 CPU oracle for the mLSTM cell forward (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``linear_rnn_mlstm_b200``) never imports it, and it imports nothing from the
product: the two share only the seeded input generator, which holds none of
the method's arithmetic.

Contents
--------
``fwd``            the sequential recurrence of "xLSTM: Extended Long Short-Term
                   Memory" section 2.3 (matrix memory, covariance rule eq. (18),
                   normaliser with lower bound 1.0) stabilised as in section 2.2,
                   in plain C float64 (``mlstm_oracle.c``), one token at a time.
``fwd_raw``        the same recurrence without the stabiliser (section 2.2 says
                   the stabilised gates leave the output unchanged; the tests
                   check that claim with this).
``step``           one decode token: ``fwd`` over S = 1 with the state carried.
``quadratic_form`` (in ``oracle.quadratic``) the parallel form that section 2.3
                   says the recurrence can be rewritten into, derived by
                   unrolling the recurrence; pure numpy, for tiny inputs.
``headnorm_gate``  (in ``oracle.headnorm``) the mLSTM block's epilogue after the
                   cell (section 2.4, Figure 10): per-head GroupNorm, learnable
                   skip, external output gate; numpy float64.
``slstm.fwd``      (in ``oracle.slstm``) the sLSTM cell of section 2.2 (scalar
                   memory, exponential gating, normaliser, stabiliser, memory
                   mixing within heads) in plain C float64 (``slstm_oracle.c``).
``grads``          (in ``oracle.backward``) gradients of a loss through the cell:
                   the recurrence in plain PyTorch float64 ops, differentiated
                   by PyTorch's reverse mode.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mlstm_oracle.c")
_LIB = os.path.join(_HERE, "libmlstm_oracle.so")
_lock = threading.Lock()
_lib = None


_SLSTM_SRC = os.path.join(_HERE, "slstm_oracle.c")
_SLSTM_LIB = os.path.join(_HERE, "libslstm_oracle.so")


def _build_one(src: str, lib: str, force: bool) -> str:
    if (not force and os.path.exists(lib)
            and os.path.getmtime(lib) >= os.path.getmtime(src)):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Compile the C oracles into ``oracle/libmlstm_oracle.so`` and
    ``oracle/libslstm_oracle.so`` (gcc, -O2, OpenMP); returns the first.

    No fast-math: the oracles keep IEEE double semantics and the source order
    of every sum.
    """
    _build_one(_SLSTM_SRC, _SLSTM_LIB, force)
    return _build_one(_SRC, _LIB, force)


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    lib.mlstm_oracle_fwd.argtypes = [dp] * 13 + [ctypes.c_long] * 3 + [ctypes.c_int] * 2
    lib.mlstm_oracle_fwd.restype = ctypes.c_int
    lib.mlstm_oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def max_threads() -> int:
    """Threads the oracle's OpenMP loop uses (OMP_NUM_THREADS or all cores)."""
    return int(_load().mlstm_oracle_max_threads())


def _f64(x, shape=None):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (any dtype) -> exact float64 copy
        x = x.detach().to("cpu").double().numpy()
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if shape is not None:
        a = a.reshape(shape)
    return a


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _run(q, k, v, i_pre, f_pre, o_pre, fgate, C0, n0, m0, stabilised, lib=None):
    q = _f64(q)
    if q.ndim != 4:
        raise ValueError("q must be [B, NH, S, DH]")
    B, NH, S, DH = q.shape
    BH = B * NH
    k = _f64(k, q.shape)
    v = _f64(v, q.shape)
    o_pre = _f64(o_pre, q.shape)
    i_pre = _f64(i_pre, (B, NH, S))
    f_pre = _f64(f_pre, (B, NH, S))
    C0 = _f64(C0, (B, NH, DH, DH))
    n0 = _f64(n0, (B, NH, DH))
    m0 = _f64(m0, (B, NH))
    h = np.empty((B, NH, S, DH), np.float64)
    C = np.empty((B, NH, DH, DH), np.float64)
    n = np.empty((B, NH, DH), np.float64)
    m = np.empty((B, NH), np.float64)
    if fgate not in ("sigmoid", "exp"):
        raise ValueError("fgate must be 'sigmoid' or 'exp'")
    rc = (lib or _load()).mlstm_oracle_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(i_pre), _ptr(f_pre), _ptr(o_pre), _ptr(h),
        _ptr(C0), _ptr(n0), _ptr(m0), _ptr(C), _ptr(n), _ptr(m),
        BH, S, DH, 1 if fgate == "exp" else 0, 1 if stabilised else 0)
    if rc != 0:
        raise MemoryError("oracle could not allocate its per-head state")
    return h, C, n, m


def fwd(q, k, v, i_pre, f_pre, o_pre, fgate="sigmoid", C0=None, n0=None, m0=None):
    """Stabilised sequential recurrence.

    Shapes: q, k, v, o_pre [B, NH, S, DH]; i_pre, f_pre [B, NH, S]; optional
    initial state C0 [B, NH, DH, DH] (row = value index, column = key index),
    n0 [B, NH, DH], m0 [B, NH] (zeros when omitted).  Inputs may be numpy
    arrays or torch tensors of any float dtype; they are converted exactly to
    float64.  Returns (h, C, n, m) as float64 numpy arrays, with the final
    state in stabilised units (C' = C exp(-m), n' = n exp(-m)).
    """
    return _run(q, k, v, i_pre, f_pre, o_pre, fgate, C0, n0, m0, True)


def fwd_raw(q, k, v, i_pre, f_pre, o_pre, fgate="sigmoid", C0=None, n0=None):
    """Unstabilised recurrence (raw units, floor 1.0).  Returns (h, C, n)."""
    h, C, n, _ = _run(q, k, v, i_pre, f_pre, o_pre, fgate, C0, n0, None, False)
    return h, C, n


def step(q, k, v, i_pre, f_pre, o_pre, C, n, m, fgate="sigmoid"):
    """One decode token for every head: q, k, v, o_pre [B, NH, DH];
    i_pre, f_pre [B, NH]; state (C, n, m) in stabilised units.
    Returns (h [B, NH, DH], C, n, m) with the updated state."""
    q = _f64(q)
    B, NH, DH = q.shape
    h, C1, n1, m1 = fwd(q.reshape(B, NH, 1, DH), _f64(k).reshape(B, NH, 1, DH),
                        _f64(v).reshape(B, NH, 1, DH), _f64(i_pre).reshape(B, NH, 1),
                        _f64(f_pre).reshape(B, NH, 1), _f64(o_pre).reshape(B, NH, 1, DH),
                        fgate, C, n, m)
    return h.reshape(B, NH, DH), C1, n1, m1


class Impl:
    """The oracle's entry points bound to a given shared library.

    ``Impl()`` is the oracle itself.  ``Impl(path)`` binds a library built from
    a deliberately altered copy of ``mlstm_oracle.c``; the tests use it to show
    that each planted mistake fails at least one pin.
    """

    def __init__(self, path=None):
        self._lib = _bind(ctypes.CDLL(path)) if path else _load()

    def fwd(self, q, k, v, i_pre, f_pre, o_pre, fgate="sigmoid", C0=None, n0=None, m0=None):
        return _run(q, k, v, i_pre, f_pre, o_pre, fgate, C0, n0, m0, True, self._lib)

    def fwd_raw(self, q, k, v, i_pre, f_pre, o_pre, fgate="sigmoid", C0=None, n0=None):
        h, C, n, _ = _run(q, k, v, i_pre, f_pre, o_pre, fgate, C0, n0, None, False, self._lib)
        return h, C, n


def build_variant(src_text: str, out_path: str) -> str:
    """Compile ``src_text`` (a copy of the oracle source) into ``out_path``."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                    "-fno-fast-math", "-ffp-contract=off", src, "-o", out_path, "-lm"],
                   check=True)
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()
