"""Pins of the float64 sLSTM oracle (``oracle.slstm``; "xLSTM: Extended Long
Short-Term Memory" section 2.2).

None of them re-types the recurrence: hand-worked steps
(``tests/golden/slstm_hand.json``, including the orientation of the recurrent
matrices and the use of the previous step's h), the running-mean special case
(no forgetting, unit input gates, no mixing), the convex-combination bound of
the normalised cell, the stated invariance under the stabiliser, continuity of
a split sequence through the carried state, and head-permutation
equivariance.  Planted mistakes in copies of the C source each fail a pin.
"""
import json
import math
import os
import tempfile

import numpy as np
import pytest

import oracle
import oracle.slstm as sl

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "slstm_hand.json")


def _val(x):
    if isinstance(x, str):
        return float(eval(x, {"__builtins__": {}}, {"ln": math.log}))
    return float(x)


def _arr(x):
    if isinstance(x, list):
        return np.array([_arr(e) for e in x], dtype=np.float64)
    return _val(x)


def _inputs(B=2, NH=3, S=9, DH=4, fgate="sigmoid", r_sd=0.5, seed=0):
    g = np.random.default_rng(seed)
    shp = (B, NH, S, DH)
    zx, ix, ox = g.normal(0, 1, shp), g.normal(0, 1, shp), g.normal(0, 1, shp)
    fx = g.normal(3, 1, shp) if fgate == "sigmoid" else g.normal(-0.05, 0.3, shp)
    R = g.normal(0, r_sd / math.sqrt(DH), (NH, 4, DH, DH))
    return zx, ix, fx, ox, R


# ------------------------------------------------------------------- pins
def pin_hand(lib=None):
    for case in json.load(open(GOLDEN))["cases"]:
        DH = case["DH"]
        S = len(case["zx"])
        x = [_arr(case[nm]).reshape(1, 1, S, DH) for nm in ("zx", "ix", "fx", "ox")]
        R = _arr(case["R"]).reshape(1, 4, DH, DH)
        h, c, n, m, hl = sl.fwd(*x, R, case["fgate"], lib_path=lib)
        np.testing.assert_allclose(h.reshape(S, DH), _arr(case["h"]), rtol=0, atol=1e-12,
                                   err_msg=case["name"])
        for nm, got in (("c", c), ("n", n), ("m", m)):
            np.testing.assert_allclose(got.reshape(DH), _arr(case[nm]), rtol=0, atol=1e-12,
                                       err_msg=f"{case['name']}: {nm}")
        np.testing.assert_allclose(hl.reshape(DH), _arr(case["h"])[-1], rtol=0, atol=1e-12)


def pin_running_mean(lib=None):
    """No forgetting (exponential forget, fx = 0), unit input gates (ix = 0),
    no mixing: the normalised cell is the running mean of z = tanh(zx)."""
    zx, _, _, ox, R = _inputs(seed=1)
    zero = np.zeros_like(zx)
    h = sl.fwd(zx, zero, zero, ox, np.zeros_like(R), "exp", lib_path=lib)[0]
    z = np.tanh(zx)
    mean = np.cumsum(z, axis=2) / np.arange(1, zx.shape[2] + 1)[None, None, :, None]
    np.testing.assert_allclose(h, mean / (1.0 + np.exp(-ox)), rtol=1e-12, atol=1e-14)


def pin_convex_combination(lib=None):
    """c_t / n_t is a weighted mean of z_1..z_t with positive weights: without
    mixing it stays within their running min and max; with mixing it stays
    inside (-1, 1) since every z = tanh(.) does."""
    for fgate in ("sigmoid", "exp"):
        zx, ix, fx, ox, R = _inputs(fgate=fgate, seed=2)
        ox_big = np.full_like(ox, 40.0)            # o = 1 to double precision
        h = sl.fwd(zx, ix, fx, ox_big, np.zeros_like(R), fgate, lib_path=lib)[0]
        z = np.tanh(zx)
        lo = np.minimum.accumulate(z, axis=2)
        hi = np.maximum.accumulate(z, axis=2)
        assert np.all(h >= lo - 1e-12) and np.all(h <= hi + 1e-12)
        h = sl.fwd(zx, ix, fx, ox_big, 4.0 * R, fgate, lib_path=lib)[0]
        assert np.all(np.abs(h) < 1.0)


def pin_stabiliser_invariance(lib=None):
    """Section 2.2: the stabilised gates leave the output unchanged."""
    for fgate in ("sigmoid", "exp"):
        x = _inputs(fgate=fgate, seed=3)
        h = sl.fwd(*x, fgate, lib_path=lib)[0]
        h_raw = sl.fwd(*x, fgate, raw=True, lib_path=lib)[0]
        np.testing.assert_allclose(h, h_raw, rtol=1e-11, atol=1e-13)


def pin_split_continuity(lib=None):
    """Running S tokens equals running the first S1 and then the rest from the
    carried state (c, n, m, h)."""
    zx, ix, fx, ox, R = _inputs(S=12, seed=4)
    full = sl.fwd(zx, ix, fx, ox, R, lib_path=lib)
    a = sl.fwd(zx[:, :, :5], ix[:, :, :5], fx[:, :, :5], ox[:, :, :5], R, lib_path=lib)
    b = sl.fwd(zx[:, :, 5:], ix[:, :, 5:], fx[:, :, 5:], ox[:, :, 5:], R, "sigmoid",
               a[1], a[2], a[3], a[4], lib_path=lib)
    np.testing.assert_allclose(np.concatenate([a[0], b[0]], axis=2), full[0], rtol=1e-12,
                               atol=1e-14)
    for i in range(1, 5):
        np.testing.assert_allclose(b[i], full[i], rtol=1e-12, atol=1e-14)


def pin_head_permutation(lib=None):
    """Mixing stays inside a head: permuting the heads (with their recurrent
    blocks) permutes the outputs."""
    zx, ix, fx, ox, R = _inputs(seed=5)
    h = sl.fwd(zx, ix, fx, ox, R, lib_path=lib)[0]
    p = np.array([2, 0, 1])
    hp = sl.fwd(zx[:, p], ix[:, p], fx[:, p], ox[:, p], R[p], lib_path=lib)[0]
    np.testing.assert_allclose(hp, h[:, p], rtol=1e-13, atol=1e-15)


PINS = [pin_hand, pin_running_mean, pin_convex_combination, pin_stabiliser_invariance,
        pin_split_continuity, pin_head_permutation]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_slstm_oracle_meets_pin(pin):
    pin()


def test_empty_sequence_passes_the_state_through():
    zx, ix, fx, ox, R = _inputs(S=0)
    st = [np.random.default_rng(6).normal(0, 1, (2, 3, 4)) for _ in range(4)]
    st[1] = np.abs(st[1]) + 0.5
    h, c, n, m, hl = sl.fwd(zx, ix, fx, ox, R, "sigmoid", *st)
    assert h.shape == (2, 3, 0, 4)
    for got, want in zip((c, n, m, hl), st):
        np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------- planted mistakes
MUTANTS = {
    "recurrent_matrix_transposed": ("zt += Rz[j * DH + l] * hp[l];", "zt += Rz[l * DH + j] * hp[l];"),
    "mixing_reads_this_step": ("                h[row + j] = hn[j];\n                hp[j] = hn[j];",
                               "                h[row + j] = hn[j];"),
    "normaliser_not_decayed": ("n[j] = fg * n[j] + ig;", "n[j] = n[j] + ig;"),
    "forget_drops_previous_m": ("fg = exp(log_f + m[j] - m_new);", "fg = exp(log_f - m_new);"),
    "no_tanh": ("const double z = tanh(zt);", "const double z = zt;"),
    "no_output_gate": ("hn[j] = o * c[j] / n[j];", "hn[j] = c[j] / n[j];"),
    "forget_activations_swapped": ("fgate_exp ? ft : log_sigmoid(ft)", "fgate_exp ? log_sigmoid(ft) : ft"),
    "input_gate_mixing_dropped": ("it += Ri[j * DH + l] * hp[l];", "it += 0.0 * hp[l];"),
    "h_updated_in_place": ("hn[j] = o * c[j] / n[j];", "hn[j] = o * c[j] / n[j]; hp[j] = hn[j];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name):
    old, new = MUTANTS[name]
    with open(os.path.join(os.path.dirname(oracle.__file__), "slstm_oracle.c")) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutant {name}: anchor not found once"
    with tempfile.TemporaryDirectory() as tmp:
        lib = oracle.build_variant(src.replace(old, new), os.path.join(tmp, f"lib_{name}.so"))
        failed = []
        for pin in PINS:
            try:
                pin(lib)
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
