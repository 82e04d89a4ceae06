"""Planted mistakes: each altered copy of the C oracle must fail at least one pin.

A copy of ``oracle/mlstm_oracle.c`` is edited by one plausible mistake (a
transposed outer product, a dropped key scaling, the floor applied in the wrong
units, a missing absolute value, a wrong stabiliser, a dropped output gate, a
sign error in log sigmoid, a wrong index), compiled on the CPU into a temporary
library and run through the same independent pins as the real oracle: the
hand-worked examples, the quadratic form, the closed-form final state and the
eq. (18) special case.  The unaltered source must pass all of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle.quadratic import quadratic_form

from test_oracle import GOLDEN, _arr, _rand_inputs, _rel, _val

MUTANTS = {
    "transposed_outer_product": ("row[j] = fg * row[j] + a * khat[j];",
                                 "row[j] = fg * row[j] + ig * khat[i] * vt[j];"),
    "no_key_scaling": ("khat[j] = kt[j] * inv_sqrt_d;", "khat[j] = kt[j];"),
    "floor_in_stabilised_units": ("floor_ = exp(-m_new);", "floor_ = 1.0;"),
    "no_abs": ("fmax(fabs(den), floor_)", "fmax(den, floor_)"),
    "stabiliser_drops_forget": ("fmax(log_f + m, log_i)", "fmax(m, log_i)"),
    "forget_drops_previous_m": ("fg = exp(log_f + m - m_new);", "fg = exp(log_f - m_new);"),
    "no_output_gate": ("ht[i] = sigmoid(ot[i]) * num / denom;", "ht[i] = num / denom;"),
    "log_sigmoid_sign": ("return -log1p(exp(-x));", "return -log1p(exp(x));"),
    "retrieval_uses_key": ("num += row[j] * qt[j];", "num += row[j] * kt[j];"),
    "normaliser_not_decayed": ("n[j] = fg * n[j] + ig * khat[j];", "n[j] = n[j] + ig * khat[j];"),
    "input_gate_not_stabilised": ("ig = exp(log_i - m_new);", "ig = exp(log_i);"),
}


def _pin_hand(impl):
    for case in json.load(open(GOLDEN))["cases"]:
        d, S = case["d"], len(case["q"])
        sh = (1, 1, S, d)
        q, k, v, o = (_arr(case[x]).reshape(sh) for x in ("q", "k", "v", "o_pre"))
        ip = _arr(case["i_pre"]).reshape(1, 1, S)
        fp = _arr(case["f_pre"]).reshape(1, 1, S)
        h, C, n, m = impl.fwd(q, k, v, ip, fp, o, case["fgate"])
        if not (np.allclose(h.reshape(S, d), _arr(case["h"]), rtol=1e-12, atol=1e-12)
                and np.allclose(C.reshape(d, d), _arr(case["C"]), rtol=1e-12, atol=1e-12)
                and abs(m.item() - _val(case["m"])) < 1e-12):
            return False
    return True


def _pin_quadratic(impl):
    for fgate, i_sd, f_mu, f_sd, seed in (("sigmoid", 1.0, 3.0, 1.0, 1), ("exp", 3.0, -0.05, 0.1, 2),
                                          ("sigmoid", 3.0, 0.0, 6.0, 3)):
        rng = np.random.default_rng(seed)
        x = _rand_inputs(rng, 1, 2, 12, 4, fgate, i_sd, f_mu, f_sd)
        h, *_ = impl.fwd(*x, fgate)
        if not _rel(h, quadratic_form(*x, fgate)) < 1e-10:
            return False
    return True


def _pin_state(impl):
    rng = np.random.default_rng(3)
    q, k, v, ip, fp, op = _rand_inputs(rng, 1, 1, 15, 4, "sigmoid", 2.0, 1.0, 2.0)
    h, C, n, m = impl.fwd(q, k, v, ip, fp, op, "sigmoid")
    F = np.cumsum(-np.logaddexp(0.0, -fp), axis=-1)[0, 0]
    w = np.exp(F[-1] - F + ip[0, 0])
    khat = k[0, 0] / 2.0
    m_ref = max(F[-1], np.max(ip[0, 0] + F[-1] - F))
    C_raw = np.einsum("s,si,sj->ij", w, v[0, 0], khat)
    return abs(m[0, 0] - m_ref) < 1e-10 and _rel(C[0, 0] * math.exp(m[0, 0]), C_raw) < 1e-10


def _pin_eq18(impl):
    rng = np.random.default_rng(7)
    q, k, v, _, _, op = _rand_inputs(rng, 1, 1, 10, 4)
    z = np.zeros((1, 1, 10))
    h, *_ = impl.fwd(q, k, v, z, z, op, "exp")
    khat = k / 2.0
    num = np.einsum("bhsij,bhsj->bhsi", np.cumsum(np.einsum("bhsi,bhsj->bhsij", v, khat), 2), q)
    den = np.maximum(np.abs(np.einsum("bhsj,bhsj->bhs", np.cumsum(khat, 2), q)), 1.0)
    return _rel(h, num / den[..., None] / (1.0 + np.exp(-op))) < 1e-10


PINS = {"hand": _pin_hand, "quadratic": _pin_quadratic, "state": _pin_state, "eq18": _pin_eq18}


def test_unaltered_oracle_passes_every_pin():
    impl = oracle.Impl()
    assert {name: pin(impl) for name, pin in PINS.items()} == {name: True for name in PINS}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = oracle.build_variant(src.replace(old, new), str(tmp_path / f"lib_{name}.so"))
    impl = oracle.Impl(path)
    with np.errstate(all="ignore"):
        results = {pname: pin(impl) for pname, pin in PINS.items()}
    assert not all(results.values()), f"mutant {name} passed every pin: {results}"
