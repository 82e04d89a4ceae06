"""Pins of the gradient oracle (``oracle.backward``): the derivative of the
mLSTM cell ("xLSTM: Extended Long Short-Term Memory" sections 2.2-2.3) taken
by reverse-mode differentiation of the plain recurrence in float64.

The pins do not re-type the recurrence: hand-worked gradients
(``tests/golden/backward_hand.json``), central finite differences of the
independent C oracle's forward, the forward itself against the C oracle, and
the pages' claim that the stabilised gates leave the loss's derivatives
unchanged (section 2.2, appendix A.2).  Planted mistakes in copies of the
module must each fail at least one pin.
"""
import json
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle
import oracle.backward as bw

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "backward_hand.json")
_SYMS = {"sqrt2": math.sqrt(2.0), "ln2": math.log(2.0)}
_KEYS = {"dq": "q", "dk": "k", "dv": "v", "di": "i_pre", "df": "f_pre", "do": "o_pre"}


def _val(x):
    if isinstance(x, str):
        return float(eval(x, {"__builtins__": {}}, dict(_SYMS)))
    return float(x)


def _arr(x):
    if x is None:
        return None
    if isinstance(x, list):
        return np.array([_arr(e) for e in x], dtype=np.float64)
    return _val(x)


def _inputs(B=1, NH=2, S=6, DH=4, fgate="sigmoid", seed=0):
    g = np.random.default_rng(seed)
    shp = (B, NH, S, DH)
    d = dict(q=g.normal(0, 1, shp), k=g.normal(0, 1, shp), v=g.normal(0, 1, shp),
             i_pre=g.normal(0, 1, shp[:3]),
             f_pre=g.normal(3, 1, shp[:3]) if fgate == "sigmoid" else g.normal(-0.3, 0.3, shp[:3]),
             o_pre=g.normal(0, 1, shp))
    dh = g.normal(0, 1, shp)
    dC = g.normal(0, 1, (B, NH, DH, DH))
    dn = g.normal(0, 1, (B, NH, DH))
    return d, dh, dC, dn


# ------------------------------------------------------------------- pins
def pin_hand(mod):
    for case in json.load(open(GOLDEN))["cases"]:
        S, d = len(case["q"]), case["d"]
        shp = (1, 1, S, d)
        args = {nm: _arr(case[nm]).reshape(shp) for nm in ("q", "k", "v", "o_pre")}
        args.update({nm: _arr(case[nm]).reshape(shp[:3]) for nm in ("i_pre", "f_pre")})
        dh = _arr(case["dh"]).reshape(shp)
        dC = None if case["dC"] is None else _arr(case["dC"]).reshape(1, 1, d, d)
        loss, g = mod.grads(args["q"], args["k"], args["v"], args["i_pre"], args["f_pre"],
                            args["o_pre"], dh, case["fgate"], dC=dC)
        assert abs(loss - case["loss"]) <= 1e-12, case["name"]
        for key, nm in _KEYS.items():
            want = _arr(case[key]).reshape(g[nm].shape)
            np.testing.assert_allclose(g[nm], want, rtol=0, atol=1e-12,
                                       err_msg=f"{case['name']}: {key}")


def pin_forward_is_the_c_oracle(mod):
    """The differentiated forward is the same function as the C oracle's."""
    for fgate in ("sigmoid", "exp"):
        d, _, _, _ = _inputs(fgate=fgate, seed=1)
        h, C, n = mod.forward(*(torch.from_numpy(d[nm]) for nm in bw.GRAD_NAMES), fgate=fgate)
        h_ref, C_ref, n_ref, _ = oracle.fwd(d["q"], d["k"], d["v"], d["i_pre"], d["f_pre"],
                                            d["o_pre"], fgate)
        np.testing.assert_allclose(h.detach().numpy(), h_ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(C.detach().numpy(), C_ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(n.detach().numpy(), n_ref, rtol=1e-12, atol=1e-13)


def _c_loss(d, dh, dC, dn, fgate):
    h, C, n, _ = oracle.fwd(d["q"], d["k"], d["v"], d["i_pre"], d["f_pre"], d["o_pre"], fgate)
    return float(np.sum(h * dh) + np.sum(C * dC) + np.sum(n * dn))


def pin_finite_differences(mod):
    """Central differences of the C oracle's loss, element by element, on a
    sample of every input (step 1e-6: truncation ~1e-12, rounding ~1e-10)."""
    eps = 1e-6
    for fgate, seed in (("sigmoid", 2), ("exp", 3)):
        d, dh, dC, dn = _inputs(fgate=fgate, seed=seed)
        _, g = mod.grads(d["q"], d["k"], d["v"], d["i_pre"], d["f_pre"], d["o_pre"], dh, fgate,
                         dC=dC, dn=dn)
        pick = np.random.default_rng(seed + 100)
        for nm in bw.GRAD_NAMES:
            flat = d[nm].reshape(-1)
            for idx in pick.choice(flat.size, size=min(8, flat.size), replace=False):
                keep = flat[idx]
                flat[idx] = keep + eps
                up = _c_loss(d, dh, dC, dn, fgate)
                flat[idx] = keep - eps
                dn_ = _c_loss(d, dh, dC, dn, fgate)
                flat[idx] = keep
                fd = (up - dn_) / (2 * eps)
                ad = g[nm].reshape(-1)[idx]
                assert abs(fd - ad) <= 1e-6 * (1.0 + abs(ad)), (fgate, nm, int(idx), fd, ad)


def pin_stabiliser_leaves_gradients_unchanged(mod):
    """Section 2.2: the stabilised gates change neither the output nor the
    derivatives of the loss (the loss on h; the returned state is in
    stabilised units by definition, so its cotangents are left out)."""
    for fgate, seed in (("sigmoid", 4), ("exp", 5)):
        d, dh, _, _ = _inputs(S=12, fgate=fgate, seed=seed)
        l_s, g_s = mod.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh, fgate)
        l_r, g_r = mod.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh, fgate, raw=True)
        assert abs(l_s - l_r) <= 1e-12 * (1 + abs(l_r))
        for nm in bw.GRAD_NAMES:
            np.testing.assert_allclose(g_s[nm], g_r[nm], rtol=1e-10, atol=1e-12, err_msg=nm)


PINS = [pin_hand, pin_forward_is_the_c_oracle, pin_finite_differences,
        pin_stabiliser_leaves_gradients_unchanged]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_gradient_oracle_meets_pin(pin):
    pin(bw)


def test_empty_sequence_and_shapes():
    d, dh, _, _ = _inputs(S=0)
    loss, g = bw.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh)
    assert loss == 0.0
    for nm in bw.GRAD_NAMES:
        assert g[nm].shape == d[nm].shape and not np.any(g[nm])


# ---------------------------------------------------------- planted mistakes
MUTANTS = {
    "output_gate_detached": ("o = torch.sigmoid(o_pre)", "o = torch.sigmoid(o_pre).detach()"),
    "input_gate_detached": ("ig = torch.exp(log_i[:, :, t] - m_new)",
                            "ig = torch.exp(log_i[:, :, t] - m_new).detach()"),
    "no_abs": ("torch.abs((n * qt).sum(-1))", "(n * qt).sum(-1)"),
    "floor_one_in_stabilised_units": ("floor = torch.exp(-m_new)",
                                      "floor = torch.ones((B, NH), dtype=torch.float64)"),
    "key_not_scaled": ("khat = k / math.sqrt(DH)", "khat = k"),
    "outer_product_transposed": ("(vt[..., :, None] * kt[..., None, :])",
                                 "(kt[..., :, None] * vt[..., None, :])"),
    "forget_drops_previous_m": ("fg = torch.exp(log_f[:, :, t] + m - m_new)",
                                "fg = torch.exp(log_f[:, :, t] - m_new)"),
    "stabiliser_ignores_forget": ("m_new = torch.maximum(log_f[:, :, t] + m, log_i[:, :, t])",
                                  "m_new = torch.maximum(m, log_i[:, :, t])"),
}


def _mutant(name):
    old, new = MUTANTS[name]
    src = open(bw.__file__).read()
    assert src.count(old) == 1, f"mutant {name}: anchor not found once"
    mod = types.ModuleType(f"backward_{name}")
    exec(compile(src.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name):
    mod = _mutant(name)
    failed = []
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"


def test_gradients_are_taken_under_no_grad_too():
    d, dh, _, _ = _inputs(seed=9)
    _, g0 = bw.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh)
    with torch.no_grad():
        _, g1 = bw.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh)
    for nm in bw.GRAD_NAMES:
        assert np.any(g1[nm]) and np.array_equal(g0[nm], g1[nm])
