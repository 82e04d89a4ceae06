"""The chunkwise backward algorithm (``tests/backward_chunkwise_model.py``, the
blocked form the gradient kernels implement) against the gradient oracle
(``oracle.backward``: reverse-mode differentiation of the plain recurrence),
on the CPU in float64: chunk sizes from 1 to larger than the sequence, ragged
tails, both forget activations, wide input gates, and final-state
cotangents."""
import numpy as np
import pytest

import oracle.backward as bw
from backward_chunkwise_model import backward as chunkwise_backward


def _inputs(B, NH, S, DH, fgate, wide=False, seed=0):
    g = np.random.default_rng(seed)
    shp = (B, NH, S, DH)
    d = dict(q=g.normal(0, 1, shp), k=g.normal(0, 1, shp), v=g.normal(0, 1, shp),
             i_pre=g.normal(0, 3 if wide else 1, shp[:3]),
             f_pre=(g.normal(3, 1, shp[:3]) if fgate == "sigmoid"
                    else g.normal(-0.05, 0.1 if not wide else 1.0, shp[:3])),
             o_pre=g.normal(0, 1, shp))
    return d, g.normal(0, 1, shp), g.normal(0, 1, (B, NH, DH, DH)), g.normal(0, 1, (B, NH, DH))


def _compare(got, ref):
    for nm in bw.GRAD_NAMES:
        scale = max(1.0, float(np.max(np.abs(ref[nm]))))
        err = float(np.max(np.abs(got[nm] - ref[nm]))) / scale
        assert err <= 1e-9, f"{nm}: max|d|/max(1,max|ref|) = {err:.3e}"


@pytest.mark.parametrize("L", [1, 3, 4, 16, 40])
@pytest.mark.parametrize("fgate", ["sigmoid", "exp"])
def test_chunkwise_backward_matches_gradient_oracle(L, fgate):
    d, dh, _, _ = _inputs(2, 2, 13, 4, fgate, seed=L)
    ref = bw.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh, fgate)[1]
    got = chunkwise_backward(*(d[nm] for nm in bw.GRAD_NAMES), dh, L, fgate)
    _compare(got, ref)


@pytest.mark.parametrize("fgate", ["sigmoid", "exp"])
def test_chunkwise_backward_wide_gates(fgate):
    """itilde ~ N(0, 3): the stabiliser moves and the floor is hit often."""
    d, dh, _, _ = _inputs(1, 3, 24, 8, fgate, wide=True, seed=7)
    ref = bw.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh, fgate)[1]
    got = chunkwise_backward(*(d[nm] for nm in bw.GRAD_NAMES), dh, 5, fgate)
    _compare(got, ref)


@pytest.mark.parametrize("fgate,wide", [("sigmoid", False), ("exp", True)])
def test_chunkwise_backward_with_final_state_cotangents(fgate, wide):
    d, dh, dC, dn = _inputs(2, 2, 11, 4, fgate, wide=wide, seed=11)
    ref = bw.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh, fgate, dC=dC, dn=dn)[1]
    got = chunkwise_backward(*(d[nm] for nm in bw.GRAD_NAMES), dh, 4, fgate, dC=dC, dn=dn)
    _compare(got, ref)


def test_chunkwise_backward_final_state_when_initial_m_is_the_maximum():
    """Input gates so small that the initial m_0 = 0 stays the stabiliser's
    maximum: the returned state's m_T then passes no gradient to any key."""
    g = np.random.default_rng(3)
    shp = (1, 2, 9, 4)
    d = dict(q=g.normal(0, 1, shp), k=g.normal(0, 1, shp), v=g.normal(0, 1, shp),
             i_pre=g.normal(-3, 0.5, shp[:3]), f_pre=np.full(shp[:3], 0.1),
             o_pre=g.normal(0, 1, shp))
    assert np.max(d["i_pre"] - np.cumsum(d["f_pre"], -1)) < 0     # m_0 is the maximum
    dh, dC, dn = g.normal(0, 1, shp), g.normal(0, 1, (1, 2, 4, 4)), g.normal(0, 1, (1, 2, 4))
    ref = bw.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh, "exp", dC=dC, dn=dn)[1]
    got = chunkwise_backward(*(d[nm] for nm in bw.GRAD_NAMES), dh, 4, "exp", dC=dC, dn=dn)
    _compare(got, ref)
