"""The sLSTM kernel's own per-unit code (``csrc/slstm_body.cuh``), run on the
CPU by a host emulation built with AddressSanitizer (units one after another
between the per-step barriers), against the float64 sLSTM oracle
(``oracle.slstm``).  The GPU parity tests then check the same code as compiled
for sm_100a.

Tolerance: max |got - ref| / max(1, max |ref|) <= 1e-5 on h and on the final
(c', n', h); m to 1e-5 absolute.  The kernel is fp32 with DH-long dot products
per gate and step; |h| < 1 and the normalised ratio c'/n' keeps the error of
each step near a few fp32 roundings.  The final c' and n' are compared
relative to their own scale (they grow like the sum of the input gates)."""
import os
import shutil
import struct
import subprocess
import tempfile

import numpy as np
import pytest

import oracle.slstm as sl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_rnn_mlstm_b200", "csrc")


@pytest.fixture(scope="module")
def emulator():
    gxx = shutil.which("g++")
    assert gxx, "g++ is needed to build the host emulation"
    tmp = tempfile.mkdtemp(prefix="slstm_emu_")
    exe = os.path.join(tmp, "slstm_emulation")
    cmd = [gxx, "-std=c++17", "-O1", "-g", "-fsanitize=address,undefined",
           "-fno-sanitize-recover=undefined", "-I", CSRC,
           os.path.join(ROOT, "tests", "slstm_emulation.cpp"), "-o", exe, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    yield exe, tmp
    shutil.rmtree(tmp, ignore_errors=True)


def inputs(B, NH, S, DH, fgate, seed, state=False):
    g = np.random.default_rng(seed)
    shp = (B, NH, S, DH)
    x = dict(zx=g.normal(0, 1, shp), ix=g.normal(0, 1, shp),
             fx=g.normal(3, 1, shp) if fgate == "sigmoid" else g.normal(-0.05, 0.3, shp),
             ox=g.normal(0, 1, shp), R=g.normal(0, 0.5 / np.sqrt(DH), (NH, 4, DH, DH)))
    x = {k: v.astype(np.float32) for k, v in x.items()}
    if state:
        st = dict(c0=g.normal(0, 1, (B, NH, DH)), n0=np.abs(g.normal(1, 0.3, (B, NH, DH))) + 0.2,
                  m0=g.normal(0, 1, (B, NH, DH)), h0=np.tanh(g.normal(0, 1, (B, NH, DH))))
        x.update({k: v.astype(np.float32) for k, v in st.items()})
    return x


def run(emulator, x, fgate):
    exe, tmp = emulator
    B, NH, S, DH = x["zx"].shape
    state = "c0" in x
    fin, fout = os.path.join(tmp, "in.bin"), os.path.join(tmp, "out.bin")
    with open(fin, "wb") as f:
        f.write(struct.pack("6i", B, NH, S, DH, 1 if fgate == "exp" else 0, state))
        for nm in ("zx", "ix", "fx", "ox", "R") + (("c0", "n0", "m0", "h0") if state else ()):
            f.write(np.ascontiguousarray(x[nm], np.float32).tobytes())
    r = subprocess.run([exe, fin, fout], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    raw = np.fromfile(fout, dtype=np.float32).astype(np.float64)
    nx, ns = B * NH * S * DH, B * NH * DH
    assert raw.size == nx + 4 * ns
    h = raw[:nx].reshape(B, NH, S, DH)
    rest = [raw[nx + i * ns: nx + (i + 1) * ns].reshape(B, NH, DH) for i in range(4)]
    return (h, *rest)


def compare(got, ref, what=("h", "c", "n", "m", "h_last")):
    for nm, g, r in zip(what, got, ref):
        if r.size == 0:
            continue
        if nm == "m":
            err = float(np.max(np.abs(g - r)))
        else:
            err = float(np.max(np.abs(g - r))) / max(1.0, float(np.max(np.abs(r))))
        assert err <= 1e-5, f"{nm}: error {err:.3e}"


def oracle_run(x, fgate):
    st = [x.get(k) for k in ("c0", "n0", "m0", "h0")]
    return sl.fwd(x["zx"], x["ix"], x["fx"], x["ox"], x["R"], fgate, *st)


CASES = [(1, 2, 17, 16, "sigmoid", False), (2, 3, 9, 8, "exp", False),
         (1, 2, 33, 48, "sigmoid", True), (1, 1, 1, 4, "exp", True), (2, 1, 0, 16, "sigmoid", True)]


@pytest.mark.parametrize("B,NH,S,DH,fgate,state", CASES,
                         ids=[f"B{c[0]}NH{c[1]}S{c[2]}DH{c[3]}-{c[4]}{'-state' if c[5] else ''}"
                              for c in CASES])
def test_slstm_unit_code_matches_oracle(emulator, B, NH, S, DH, fgate, state):
    x = inputs(B, NH, S, DH, fgate, seed=S + DH, state=state)
    compare(run(emulator, x, fgate), oracle_run(x, fgate))


def test_slstm_unit_code_growing_forget_and_wide_input_gates(emulator):
    """Exponential forget above 1 and input gates ~ N(0, 3): the raw state would
    grow without bound; the stabilised one does not, and h stays a mean."""
    x = inputs(1, 2, 64, 16, "exp", seed=12)
    g = np.random.default_rng(13)
    x["fx"] = g.normal(0.3, 0.2, x["fx"].shape).astype(np.float32)
    x["ix"] = g.normal(0.0, 3.0, x["ix"].shape).astype(np.float32)
    compare(run(emulator, x, "exp"), oracle_run(x, "exp"))
