"""Pins of the block-epilogue oracle (``oracle.headnorm``): per-head GroupNorm,
learnable skip and external output gate ("xLSTM: Extended Long Short-Term
Memory" section 2.4, Figure 10; GroupNorm as defined by Wu & He).

Nothing here re-types the oracle's formula.  The pins are hand-worked values
(``tests/golden/headnorm_hand.json``), torch's own float64 GroupNorm and
LayerNorm (the library routines the pages' description reduces to), the exact
invariances of a normalisation (scale and shift of a head's row, with eps
scaled along), identities of the two gate activations, and equivariance under
head and token permutations.  Planted mistakes in copies of the oracle's source
must each fail at least one pin.
"""
import json
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle.headnorm as hn

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "headnorm_hand.json")
_SYMS = {"ln3": math.log(3)}


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


def _inputs(B=2, NH=3, S=5, DH=8, seed=0):
    g = np.random.default_rng(seed)
    D = NH * DH
    return dict(h=g.normal(0.3, 1.7, (B, NH, S, DH)), gamma=g.normal(1.0, 0.5, D),
                beta=g.normal(0.0, 0.5, D), skip_w=g.normal(0.0, 1.0, D),
                x_skip=g.normal(0.0, 1.0, (B, S, D)), z=g.normal(0.0, 2.0, (B, S, D)))


# ------------------------------------------------------------------- pins
def pin_hand(fn):
    for case in json.load(open(GOLDEN))["cases"]:
        y = fn(_arr(case["h"]), _arr(case["gamma"]), _arr(case["beta"]), _arr(case["z"]),
               _arr(case["skip_w"]), _arr(case["x_skip"]), eps=case["eps"], ogate=case["ogate"])
        np.testing.assert_allclose(y, _arr(case["y"]), rtol=0, atol=1e-12, err_msg=case["name"])


def pin_torch_group_norm(fn):
    """No skip and a gate of exactly 1 (sigmoid of +inf): the op is GroupNorm
    with NH groups over the NH*DH channels of each token, and equally a
    LayerNorm over each head's DH channels."""
    d = _inputs()
    B, NH, S, DH = d["h"].shape
    one = np.full((B, S, NH * DH), np.inf)
    y = fn(d["h"], d["gamma"], d["beta"], one, eps=0.3, ogate="sigmoid")
    x = torch.from_numpy(d["h"]).permute(0, 2, 1, 3).reshape(B * S, NH * DH)
    ref = torch.nn.functional.group_norm(x, NH, torch.from_numpy(d["gamma"]),
                                         torch.from_numpy(d["beta"]), eps=0.3)
    np.testing.assert_allclose(y.reshape(B * S, NH * DH), ref.numpy(), rtol=1e-12, atol=1e-12)
    ln = torch.nn.functional.layer_norm(x.reshape(B * S, NH, DH), (DH,), eps=0.3)
    ln = ln.reshape(B * S, NH * DH) * torch.from_numpy(d["gamma"]) + torch.from_numpy(d["beta"])
    np.testing.assert_allclose(y.reshape(B * S, NH * DH), ln.numpy(), rtol=1e-12, atol=1e-12)


def pin_scale_shift(fn):
    """(x - mean)/sqrt(var + eps) is unchanged when each head's row becomes
    a x + c (a > 0) and eps becomes a^2 eps."""
    d = _inputs(seed=1)
    B, NH, S, DH = d["h"].shape
    g = np.random.default_rng(11)
    a = g.uniform(0.5, 4.0, (B, NH, S, 1))
    c = g.normal(0.0, 3.0, (B, NH, S, 1))
    y0 = fn(d["h"], d["gamma"], d["beta"], d["z"], d["skip_w"], d["x_skip"], eps=0.2)
    # one eps for the whole call: scale every row by the same a
    y1 = fn(2.5 * d["h"] + c, d["gamma"], d["beta"], d["z"], d["skip_w"], d["x_skip"],
            eps=0.2 * 2.5 ** 2)
    np.testing.assert_allclose(y1, y0, rtol=1e-10, atol=1e-12)
    # eps -> 0 limit: rows scaled independently give the same output
    y2 = fn(a * d["h"] + c, d["gamma"], d["beta"], d["z"], d["skip_w"], d["x_skip"], eps=1e-30)
    y3 = fn(d["h"], d["gamma"], d["beta"], d["z"], d["skip_w"], d["x_skip"], eps=1e-30)
    np.testing.assert_allclose(y2, y3, rtol=1e-9, atol=1e-12)


def pin_gates(fn):
    """sigmoid(z) + sigmoid(-z) = 1 and silu(z) - silu(-z) = z, through the
    whole op (the ungated value is the output with a gate of exactly 1)."""
    d = _inputs(seed=2)
    args = (d["h"], d["gamma"], d["beta"])
    skip = dict(skip_w=d["skip_w"], x_skip=d["x_skip"], eps=0.1)
    base = fn(*args, np.full_like(d["z"], np.inf), ogate="sigmoid", **skip)
    sp = fn(*args, d["z"], ogate="sigmoid", **skip)
    sm = fn(*args, -d["z"], ogate="sigmoid", **skip)
    np.testing.assert_allclose(sp + sm, base, rtol=1e-12, atol=1e-12)
    lp = fn(*args, d["z"], ogate="silu", **skip)
    lm = fn(*args, -d["z"], ogate="silu", **skip)
    np.testing.assert_allclose(lp - lm, d["z"] * base, rtol=1e-10, atol=1e-12)
    # the skip term is not normalised: doubling x_skip adds skip_w * x_skip * gate once more
    two = fn(*args, d["z"], ogate="sigmoid", skip_w=d["skip_w"], x_skip=2 * d["x_skip"], eps=0.1)
    sig = 1.0 / (1.0 + np.exp(-d["z"]))
    np.testing.assert_allclose(two - sp, d["skip_w"] * d["x_skip"] * sig, rtol=1e-10, atol=1e-12)


def pin_permutations(fn):
    """Heads are independent groups and tokens independent samples: permuting
    heads (with their channel blocks of every per-channel input) or tokens
    permutes the output the same way."""
    d = _inputs(seed=3)
    B, NH, S, DH = d["h"].shape
    y = fn(d["h"], d["gamma"], d["beta"], d["z"], d["skip_w"], d["x_skip"], eps=0.05)
    perm = np.array([2, 0, 1])
    ch = (perm[:, None] * DH + np.arange(DH)[None, :]).reshape(-1)
    yp = fn(d["h"][:, perm], d["gamma"][ch], d["beta"][ch], d["z"][..., ch], d["skip_w"][ch],
            d["x_skip"][..., ch], eps=0.05)
    np.testing.assert_allclose(yp, y[..., ch], rtol=1e-12, atol=1e-12)
    tp = np.array([4, 2, 0, 3, 1])
    yt = fn(d["h"][:, :, tp], d["gamma"], d["beta"], d["z"][:, tp], d["skip_w"],
            d["x_skip"][:, tp], eps=0.05)
    np.testing.assert_allclose(yt, y[:, tp], rtol=1e-12, atol=1e-12)


PINS = [pin_hand, pin_torch_group_norm, pin_scale_shift, pin_gates, pin_permutations]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_meets_pin(pin):
    pin(hn.headnorm_gate)


def test_argument_checks():
    d = _inputs()
    with pytest.raises(ValueError):
        hn.headnorm_gate(d["h"], d["gamma"], d["beta"], d["z"], d["skip_w"], None)
    with pytest.raises(ValueError):
        hn.headnorm_gate(d["h"], d["gamma"], d["beta"], d["z"], eps=0.0)
    with pytest.raises(ValueError):
        hn.headnorm_gate(d["h"], d["gamma"], d["beta"], d["z"], ogate="tanh")


# ---------------------------------------------------------- planted mistakes
MUTANTS = {
    "unbiased_variance": ("((x - mean) ** 2).mean(axis=3, keepdims=True)",
                          "((x - mean) ** 2).sum(axis=3, keepdims=True) / (DH - 1)"),
    "heads_not_transposed": ("x = h.transpose(0, 2, 1, 3)", "x = h.reshape(B, S, NH, DH)"),
    "eps_outside_sqrt": ("np.sqrt(var + eps)", "(np.sqrt(var) + eps)"),
    "normalised_over_heads": ("mean = x.mean(axis=3, keepdims=True)",
                              "mean = x.mean(axis=2, keepdims=True)"),
    "skip_not_weighted": ("_f64(skip_w) * _f64(x_skip)", "_f64(x_skip)"),
    "beta_inside_scale": ("* _f64(gamma) + _f64(beta)", "* (_f64(gamma) + _f64(beta))"),
    "silu_drops_z": ("return z * sig", "return sig"),
    "sigmoid_sign": ("np.exp(-z)", "np.exp(z)"),
    "skip_after_gate": ("    return y * gate(_f64(z).reshape(B, S, NH * DH), ogate)",
                        "    g = gate(_f64(z).reshape(B, S, NH * DH), ogate)\n"
                        "    if skip_w is not None:\n"
                        "        return (y - _f64(skip_w) * _f64(x_skip).reshape(B, S, NH * DH)) * g"
                        " + _f64(skip_w) * _f64(x_skip).reshape(B, S, NH * DH)\n"
                        "    return y * g"),
}


def _mutant(name):
    old, new = MUTANTS[name]
    src = open(hn.__file__).read()
    assert src.count(old) == 1, f"mutant {name}: anchor not found once"
    mod = types.ModuleType(f"headnorm_{name}")
    exec(compile(src.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
    return mod.headnorm_gate


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name):
    fn = _mutant(name)
    failed = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(fn)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
