"""Pins for the float64 oracle, against what the pages and the mathematics fix.

Every check here is independent of the oracle's own code: hand-worked values
(``golden/hand_examples.json``), the quadratic form derived by unrolling the
recurrence, the stabiliser invariance claimed in "xLSTM: Extended Long
Short-Term Memory" section 2.2 / appendix A.2, the eq. (18) special case
(normalised causal linear attention via cumulative sums), a memoryless special
case, the closed form of the stabiliser, the floor of section 2.3, head
independence (section 2.3: heads have no memory mixing) and split continuity
(linear time, constant memory: section 2.5).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle.quadratic import quadratic_form

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")
_SYMS = {"ln2": math.log(2), "ln3": math.log(3), "ln4": math.log(4),
         "-ln2": -math.log(2), "-ln3": -math.log(3), "sqrt2": math.sqrt(2)}


def _val(x):
    if isinstance(x, str):
        if x in _SYMS:
            return _SYMS[x]
        if "/" in x:
            a, b = x.split("/")
            return float(a) / float(b)
        raise ValueError(x)
    return float(x)


def _arr(x):
    return np.vectorize(_val, otypes=[float])(np.array(x, dtype=object))


def _rand_inputs(rng, B, NH, S, DH, fgate="sigmoid", i_sd=1.0, f_mu=3.0, f_sd=1.0):
    q = rng.standard_normal((B, NH, S, DH))
    k = rng.standard_normal((B, NH, S, DH))
    v = rng.standard_normal((B, NH, S, DH))
    i_pre = rng.standard_normal((B, NH, S)) * i_sd
    f_pre = rng.standard_normal((B, NH, S)) * f_sd + f_mu
    o_pre = rng.standard_normal((B, NH, S, DH))
    return q, k, v, i_pre, f_pre, o_pre


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# ---------------------------------------------------------------- hand values
@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_worked_examples(case):
    d = case["d"]
    S = len(case["q"])
    sh = (1, 1, S, d)
    q, k, v, o = (_arr(case[x]).reshape(sh) for x in ("q", "k", "v", "o_pre"))
    i_pre = _arr(case["i_pre"]).reshape(1, 1, S)
    f_pre = _arr(case["f_pre"]).reshape(1, 1, S)
    h, C, n, m = oracle.fwd(q, k, v, i_pre, f_pre, o, case["fgate"])
    np.testing.assert_allclose(h.reshape(S, d), _arr(case["h"]), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(C.reshape(d, d), _arr(case["C"]), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(n.reshape(d), _arr(case["n"]), rtol=1e-14, atol=1e-14)
    assert abs(m.item() - _val(case["m"])) < 1e-14
    # the raw recurrence gives the same output (section 2.2: f', i' leave it unchanged)
    hr, Cr, nr = oracle.fwd_raw(q, k, v, i_pre, f_pre, o, case["fgate"])
    np.testing.assert_allclose(hr.reshape(S, d), _arr(case["h"]), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(Cr.reshape(d, d), _arr(case["C"]) * math.exp(_val(case["m"])),
                               rtol=1e-14, atol=1e-14)


# ------------------------------------------------------ quadratic (parallel) form
@pytest.mark.parametrize("regime", [
    dict(fgate="sigmoid", i_sd=1.0, f_mu=3.0, f_sd=1.0),
    dict(fgate="exp", i_sd=3.0, f_mu=-0.05, f_sd=0.1),
    dict(fgate="sigmoid", i_sd=3.0, f_mu=0.0, f_sd=6.0),     # both log-sigmoid branches
    dict(fgate="sigmoid", i_sd=1.0, f_mu=-2.0, f_sd=1.0),    # strong forgetting
])
@pytest.mark.parametrize("shape", [(1, 1, 1, 2), (2, 3, 7, 4), (1, 2, 16, 8), (1, 1, 13, 5)])
def test_recurrence_equals_quadratic_form(regime, shape):
    rng = np.random.default_rng(hash((tuple(shape), regime["fgate"], regime["f_mu"])) % 2**32)
    q, k, v, ip, fp, op = _rand_inputs(rng, *shape, **regime)
    h, *_ = oracle.fwd(q, k, v, ip, fp, op, regime["fgate"])
    hq = quadratic_form(q, k, v, ip, fp, op, regime["fgate"])
    assert _rel(h, hq) < 1e-12


# ---------------------------------------------------------------- invariance
@pytest.mark.parametrize("fgate,i_sd,f_mu,f_sd", [("sigmoid", 1.0, 3.0, 1.0),
                                                 ("exp", 3.0, -0.05, 0.1),
                                                 ("sigmoid", 4.0, 1.0, 3.0)])
def test_stabiliser_leaves_output_unchanged(fgate, i_sd, f_mu, f_sd):
    rng = np.random.default_rng(11)
    q, k, v, ip, fp, op = _rand_inputs(rng, 2, 2, 48, 8, fgate, i_sd, f_mu, f_sd)
    h, C, n, m = oracle.fwd(q, k, v, ip, fp, op, fgate)
    hr, Cr, nr = oracle.fwd_raw(q, k, v, ip, fp, op, fgate)
    assert _rel(h, hr) < 1e-12
    # stabilised state times exp(m) is the raw state
    assert _rel(C * np.exp(m)[..., None, None], Cr) < 1e-12
    assert _rel(n * np.exp(m)[..., None], nr) < 1e-12


def test_output_independent_of_initial_stabiliser():
    """Shifting (C0, n0, m0) to (C0 e^-c, n0 e^-c, m0 + c) describes the same raw
    state; the output must not change (the floor scales with the state)."""
    rng = np.random.default_rng(5)
    q, k, v, ip, fp, op = _rand_inputs(rng, 1, 2, 20, 6)
    C0 = rng.standard_normal((1, 2, 6, 6))
    n0 = rng.standard_normal((1, 2, 6))
    m0 = np.array([[0.3, -1.2]])
    h1, *_ = oracle.fwd(q, k, v, ip, fp, op, "sigmoid", C0, n0, m0)
    c = 2.5
    h2, *_ = oracle.fwd(q, k, v, ip, fp, op, "sigmoid", C0 * math.exp(-c), n0 * math.exp(-c), m0 + c)
    assert _rel(h1, h2) < 1e-12


# ------------------------------------------------ closed forms and special cases
def test_final_state_closed_form():
    """C'_T = exp(-m_T) sum_s exp(F_T - F_s + itilde_s) v_s khat_s^T, row = value."""
    rng = np.random.default_rng(3)
    B, NH, S, D = 1, 2, 30, 5
    q, k, v, ip, fp, op = _rand_inputs(rng, B, NH, S, D, "sigmoid", 2.0, 1.0, 2.0)
    h, C, n, m = oracle.fwd(q, k, v, ip, fp, op, "sigmoid")
    lf = -np.logaddexp(0.0, -fp)
    F = np.cumsum(lf, axis=-1)
    for hh in range(NH):
        w = np.exp(F[0, hh, -1] - F[0, hh] + ip[0, hh])             # [S]
        khat = k[0, hh] / math.sqrt(D)
        C_raw = np.einsum("s,si,sj->ij", w, v[0, hh], khat)
        n_raw = np.einsum("s,sj->j", w, khat)
        # m closed form: m_T = max(m_0 + F_T, max_s(itilde_s + F_T - F_s)), m_0 = 0
        m_ref = max(F[0, hh, -1], np.max(ip[0, hh] + F[0, hh, -1] - F[0, hh]))
        assert abs(m[0, hh] - m_ref) < 1e-12
        assert _rel(C[0, hh] * math.exp(m[0, hh]), C_raw) < 1e-12
        assert _rel(n[0, hh] * math.exp(m[0, hh]), n_raw) < 1e-12


def test_eq18_special_case_is_causal_linear_attention():
    """f = i = 1 reduces the gated rule to eq. (18), C_t = C_{t-1} + v_t khat_t^T:
    h~ is then causal linear attention normalised by max(|sum_s q_t.khat_s|, 1)."""
    rng = np.random.default_rng(7)
    B, NH, S, D = 1, 3, 25, 6
    q, k, v, _, _, op = _rand_inputs(rng, B, NH, S, D)
    zeros = np.zeros((B, NH, S))
    h, *_ = oracle.fwd(q, k, v, zeros, zeros, op, "exp")
    khat = k / math.sqrt(D)
    Ccum = np.cumsum(np.einsum("bhsi,bhsj->bhsij", v, khat), axis=2)
    ncum = np.cumsum(khat, axis=2)
    num = np.einsum("bhsij,bhsj->bhsi", Ccum, q)
    den = np.maximum(np.abs(np.einsum("bhsj,bhsj->bhs", ncum, q)), 1.0)
    ref = (1.0 / (1.0 + np.exp(-op))) * num / den[..., None]
    assert _rel(h, ref) < 1e-12


def test_memoryless_special_case():
    """With log f = -1e4 every token forgets the past: the 1-step closed form
    h~_t = e^{i_t} (khat_t.q_t) v_t / max(e^{i_t} |khat_t.q_t|, 1) holds at each t."""
    rng = np.random.default_rng(9)
    B, NH, S, D = 2, 1, 17, 4
    q, k, v, ip, _, op = _rand_inputs(rng, B, NH, S, D, i_sd=2.0)
    fp = np.full((B, NH, S), -1e4)
    h, *_ = oracle.fwd(q, k, v, ip, fp, op, "exp")
    kq = np.einsum("bhsd,bhsd->bhs", k / math.sqrt(D), q)
    num = (np.exp(ip) * kq)[..., None] * v
    den = np.maximum(np.exp(ip) * np.abs(kq), 1.0)[..., None]
    ref = num / den / (1.0 + np.exp(-op))
    assert _rel(h, ref) < 1e-12


def test_log_sigmoid_gate_matches_exponential_gate_on_log_sigmoid():
    """The sigmoid forget gate equals the exponential gate fed log sigmoid(ftilde),
    across both branches and far tails of log sigmoid (section 2.2 allows either)."""
    rng = np.random.default_rng(13)
    q, k, v, ip, fp, op = _rand_inputs(rng, 1, 2, 40, 4, f_mu=0.0, f_sd=20.0)
    h1, C1, n1, m1 = oracle.fwd(q, k, v, ip, fp, op, "sigmoid")
    h2, C2, n2, m2 = oracle.fwd(q, k, v, ip, -np.logaddexp(0.0, -fp), op, "exp")
    assert _rel(h1, h2) < 1e-12 and _rel(C1, C2) < 1e-12 and np.max(np.abs(m1 - m2)) < 1e-12


def test_floor_bound():
    """Section 2.3: the denominator is |n^T q| floored at 1.0 in raw units, so
    |h~_j| <= |(C_t q_t)_j| elementwise; equality when |n^T q| <= 1."""
    rng = np.random.default_rng(17)
    q, k, v, ip, fp, op = _rand_inputs(rng, 1, 1, 40, 6, "sigmoid", 2.0, 2.0, 1.0)
    op = np.full_like(op, 50.0)                      # o ~ 1 so h ~ h~
    h, *_ = oracle.fwd(q, k, v, ip, fp, op, "sigmoid")
    lf = -np.logaddexp(0.0, -fp)
    F = np.cumsum(lf, axis=-1)[0, 0]
    khat = k[0, 0] / math.sqrt(6)
    hit = 0
    for t in range(40):
        w = np.exp(F[t] - F[:t + 1] + ip[0, 0, :t + 1])
        Cq = np.einsum("s,si,s->i", w, v[0, 0, :t + 1], khat[:t + 1] @ q[0, 0, t])
        nq = float(np.sum(w * (khat[:t + 1] @ q[0, 0, t])))
        assert np.all(np.abs(h[0, 0, t]) <= np.abs(Cq) * (1 + 1e-12) + 1e-300)
        if abs(nq) <= 1.0:
            hit += 1
            assert _rel(h[0, 0, t], Cq) < 1e-12
        else:
            assert _rel(h[0, 0, t], Cq / abs(nq)) < 1e-12
    assert hit > 0


# ------------------------------------------------------- symmetry and splitting
def test_heads_and_batches_are_independent():
    rng = np.random.default_rng(19)
    q, k, v, ip, fp, op = _rand_inputs(rng, 3, 4, 12, 4)
    h, C, n, m = oracle.fwd(q, k, v, ip, fp, op)
    pb, ph = np.array([2, 0, 1]), np.array([3, 1, 0, 2])
    P = lambda x: x[pb][:, ph]
    h2, C2, n2, m2 = oracle.fwd(P(q), P(k), P(v), P(ip), P(fp), P(op))
    assert np.array_equal(h2, P(h)) and np.array_equal(C2, P(C)) and np.array_equal(m2, P(m))


def test_split_continuity_fwd_fwd_and_fwd_steps():
    """Section 2.5: linear time, constant memory -- the state carries everything."""
    rng = np.random.default_rng(23)
    q, k, v, ip, fp, op = _rand_inputs(rng, 2, 2, 33, 5, "sigmoid", 2.0, 2.0, 1.5)
    h, C, n, m = oracle.fwd(q, k, v, ip, fp, op)
    s1 = 20
    cut = lambda x, a, b: x[:, :, a:b]
    ha, Ca, na, ma = oracle.fwd(*(cut(x, 0, s1) for x in (q, k, v, ip, fp, op)))
    hb, Cb, nb, mb = oracle.fwd(*(cut(x, s1, 33) for x in (q, k, v, ip, fp, op)), "sigmoid", Ca, na, ma)
    assert _rel(np.concatenate([ha, hb], 2), h) < 1e-12
    assert _rel(Cb, C) < 1e-12 and _rel(nb, n) < 1e-12 and np.max(np.abs(mb - m)) < 1e-12
    Cs, ns, ms = Ca, na, ma
    for t in range(s1, 33):
        ht, Cs, ns, ms = oracle.step(q[:, :, t], k[:, :, t], v[:, :, t], ip[:, :, t],
                                     fp[:, :, t], op[:, :, t], Cs, ns, ms)
        assert _rel(ht, h[:, :, t]) < 1e-12
    assert _rel(Cs, C) < 1e-12


def test_empty_sequence_returns_initial_state():
    rng = np.random.default_rng(29)
    B, NH, D = 1, 2, 4
    e = np.zeros((B, NH, 0, D))
    C0 = rng.standard_normal((B, NH, D, D))
    n0 = rng.standard_normal((B, NH, D))
    m0 = rng.standard_normal((B, NH))
    h, C, n, m = oracle.fwd(e, e, e, e[..., 0], e[..., 0], e, "sigmoid", C0, n0, m0)
    assert h.shape == (B, NH, 0, D)
    assert np.array_equal(C, C0) and np.array_equal(n, n0) and np.array_equal(m, m0)
