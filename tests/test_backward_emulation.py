"""The backward kernels' own per-thread code (``csrc/bwd_body.cuh``), run on
the CPU by a host emulation built with AddressSanitizer, against the float64
gradient oracle (``oracle.backward``).  This checks the kernels' arithmetic and
that every access stays inside the buffers they are given, before the kernels
run on a GPU; the GPU parity tests then check the same code as compiled for
sm_100a.

Tolerance, per gradient tensor, max |got - ref| / max(1, max |ref|): 1e-4, and
5e-4 for wide input gates (itilde ~ N(0, 3)) with the exponential forget gate.
The kernels work in fp32; evaluating the definition itself in fp32 (the
oracle's recurrence and reverse mode run in float32 instead of float64) gives
~1e-6 on these inputs, but 1.7e-4 on the wide-gate case, where each
stabilised exponent is formed from fp32 numbers of magnitude ~10 and the
error compounds along the sequence (the same effect as the forward's fp32
tolerance for wide gates)."""
import os
import shutil
import struct
import subprocess
import tempfile

import numpy as np
import pytest

import oracle.backward as bw

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_rnn_mlstm_b200", "csrc")
CUDA_INC = "/usr/local/cuda/include"
NAMES = ("q", "k", "v", "i_pre", "f_pre", "o_pre")


@pytest.fixture(scope="module")
def emulator():
    gxx = shutil.which("g++")
    assert gxx, "g++ is needed to build the host emulation"
    tmp = tempfile.mkdtemp(prefix="bwd_emu_")
    exe = os.path.join(tmp, "bwd_emulation")
    cmd = [gxx, "-std=c++17", "-O1", "-g", "-fsanitize=address,undefined",
           "-fno-sanitize-recover=undefined", "-I", CSRC, "-I", CUDA_INC,
           os.path.join(ROOT, "tests", "bwd_emulation.cpp"), "-o", exe, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    yield exe, tmp
    shutil.rmtree(tmp, ignore_errors=True)


def _inputs(B, NH, S, DH, fgate, wide, seed):
    g = np.random.default_rng(seed)
    shp = (B, NH, S, DH)
    d = dict(q=g.normal(0, 1, shp), k=g.normal(0, 1, shp), v=g.normal(0, 1, shp),
             i_pre=g.normal(0, 3 if wide else 1, shp[:3]),
             f_pre=(g.normal(3, 1, shp[:3]) if fgate == "sigmoid"
                    else g.normal(-0.05, 1.0 if wide else 0.1, shp[:3])),
             o_pre=g.normal(0, 1, shp))
    d = {nm: x.astype(np.float32) for nm, x in d.items()}
    dh = g.normal(0, 1, shp).astype(np.float32)
    dC = g.normal(0, 1, (B, NH, DH, DH)).astype(np.float32)
    dn = g.normal(0, 1, (B, NH, DH)).astype(np.float32)
    return d, dh, dC, dn


def _run(emulator, d, dh, L, fgate, dC=None, dn=None):
    exe, tmp = emulator
    B, NH, S, DH = d["q"].shape
    fin, fout = os.path.join(tmp, "in.bin"), os.path.join(tmp, "out.bin")
    with open(fin, "wb") as f:
        f.write(struct.pack("8i", B, NH, S, DH, L, 1 if fgate == "exp" else 0,
                            dC is not None, dn is not None))
        for nm in ("q", "k", "v", "i_pre", "f_pre", "o_pre"):
            f.write(np.ascontiguousarray(d[nm], np.float32).tobytes())
        f.write(np.ascontiguousarray(dh, np.float32).tobytes())
        for a in (dC, dn):
            if a is not None:
                f.write(np.ascontiguousarray(a, np.float32).tobytes())
    r = subprocess.run([exe, fin, fout], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    raw = np.fromfile(fout, dtype=np.float32)
    nx, ng = B * NH * S * DH, B * NH * S
    sizes = [nx, nx, nx, ng, ng, nx]
    shapes = [(B, NH, S, DH)] * 3 + [(B, NH, S)] * 2 + [(B, NH, S, DH)]
    out, off = {}, 0
    for nm, n, shp in zip(NAMES, sizes, shapes):
        out[nm] = raw[off:off + n].reshape(shp).astype(np.float64)
        off += n
    assert off == raw.size
    return out


def _compare(got, ref, tol):
    for nm in NAMES:
        scale = max(1.0, float(np.max(np.abs(ref[nm])))) if ref[nm].size else 1.0
        err = float(np.max(np.abs(got[nm] - ref[nm]))) / scale if ref[nm].size else 0.0
        assert err <= tol, f"d{nm}: max|d|/max(1,max|ref|) = {err:.3e} (tol {tol})"


CASES = [
    # B, NH, S, DH, L, fgate, wide, cotangents
    (1, 2, 13, 16, 4, "sigmoid", False, False),
    (2, 1, 13, 16, 1, "exp", False, False),
    (1, 2, 21, 32, 8, "exp", True, False),
    (2, 2, 17, 16, 64, "sigmoid", False, True),
    (1, 1, 40, 16, 16, "exp", True, True),
    (1, 1, 1, 16, 4, "sigmoid", False, True),
    (1, 1, 10, 48, 3, "sigmoid", False, True),
]


@pytest.mark.parametrize("B,NH,S,DH,L,fgate,wide,cot", CASES,
                         ids=[f"B{c[0]}NH{c[1]}S{c[2]}DH{c[3]}L{c[4]}-{c[5]}{'-wide' if c[6] else ''}"
                              f"{'-cot' if c[7] else ''}" for c in CASES])
def test_backward_kernel_bodies_match_gradient_oracle(emulator, B, NH, S, DH, L, fgate, wide, cot):
    d, dh, dC, dn = _inputs(B, NH, S, DH, fgate, wide, seed=S * 7 + DH + L)
    kw = dict(dC=dC, dn=dn) if cot else {}
    ref = bw.grads(*(d[nm] for nm in NAMES), dh, fgate, **kw)[1]
    got = _run(emulator, d, dh, L, fgate, **kw)
    _compare(got, ref, 5e-4 if wide else 1e-4)


def test_backward_kernel_bodies_floor_dominated(emulator):
    """Input gates so small (itilde ~ N(-4, 1)) that the normaliser's floor is
    active on every token of this draw: dnq' = 0 throughout, the floor passes
    no gradient, and only the numerator's terms carry one."""
    d, dh, dC, dn = _inputs(1, 2, 30, 16, "sigmoid", False, seed=5)
    g = np.random.default_rng(6)
    d["i_pre"] = g.normal(-4, 1, d["i_pre"].shape).astype(np.float32)
    ref = bw.grads(*(d[nm] for nm in NAMES), dh, "sigmoid", dC=dC, dn=dn)[1]
    got = _run(emulator, d, dh, 8, "sigmoid", dC=dC, dn=dn)
    _compare(got, ref, 1e-4)


def test_backward_kernel_bodies_growing_forget(emulator):
    """Exponential forget gate above 1 (ftilde ~ N(0.3, 0.2)): the state grows
    along the sequence and the stabiliser carries the scale."""
    d, dh, _, _ = _inputs(1, 1, 48, 16, "exp", False, seed=8)
    g = np.random.default_rng(9)
    d["f_pre"] = g.normal(0.3, 0.2, d["f_pre"].shape).astype(np.float32)
    ref = bw.grads(*(d[nm] for nm in NAMES), dh, "exp")[1]
    got = _run(emulator, d, dh, 16, "exp")
    _compare(got, ref, 5e-4)


def test_backward_kernel_bodies_empty_sequence(emulator):
    d, dh, _, _ = _inputs(1, 2, 0, 16, "sigmoid", False, seed=1)
    got = _run(emulator, d, dh, 8, "sigmoid")
    assert all(got[nm].size == 0 for nm in NAMES)
