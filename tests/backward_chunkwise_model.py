"""The blocked (chunkwise) backward of the mLSTM cell, in float64 numpy: the
algorithm the gradient kernels implement, written plainly so that it can be
checked against the gradient oracle on the CPU.  It is neither the oracle (it
chunks, reorders and works in stabilised units) nor the product.

Per head, with chunk-local cumulative log forget b, stabiliser m_t and the
forward's stabilised quantities recomputed chunk by chunk (num'_t = C'_t q_t,
nq'_t = n'_t . q_t, den'_t = max(|nq'_t|, e^{-m_t}), h~ = num'/den'):

  dnum'_t = dh~_t / den'_t,   dnq'_t = -(dh~_t . h~_t) / den'_t * sign(nq'_t)
            [only where |nq'_t| > e^{-m_t}; the floor passes no gradient]

and everything else follows from the raw recurrence with the stabiliser held
fixed ("xLSTM: Extended Long Short-Term Memory" section 2.2: the stabilised
gates change neither the output nor the loss's derivatives):

  * a reverse state dC~ (value x key) and dn~, stabilised at the chunk end's m,
    carried from the last chunk to the first:
        dC~_{c-1} = e^{B_c + m_{c-1} - m_c} dC~_c + sum_{t in c} g_t dnum'_t q_t^T,
        g_t = e^{b_t + m_{c-1} - m_t}  (the forward's decay of the incoming state);
  * per chunk, intra weights W_ts = e^{b_t - b_s + itilde_s - m_t} (s <= t),
    dP_ts = dnum'_t . v_s + dnq'_t, and
        dq   = (W o dP) khat + g (C'_prev^T dnum' + dnq' n'_prev),
        dkhat = (W o dP)^T q + wk (dC~^T v + dn~),   wk_s = e^{B - b_s + itilde_s - m_end},
        dv   = (W o S)^T dnum' + wk (dC~ khat),     S_ts = q_t . khat_s;
  * ditilde_s = khat_s . dkhat_s (each term of dkhat_s carries the input gate
    of key s once);
  * d log f_j = sum_{t >= j} (A_t - B_t), with A_t = dnum'_t . num'_t +
    dnq'_t nq'_t (what token t's output owes to its cumulative decay) and
    B_t = ditilde_t (what key t's contributions owe to it);
  * final-state cotangents dC', dn' seed the reverse state; the returned state
    is stabilised by m_T = F_T + max(m_0, max_s(itilde_s - F_s)), so its
    explicit dependence on m_T adds -A_final (A_final = sum dC' o C'_T +
    sum dn' o n'_T) to itilde_{s*} and +A_final to F_{s*} for the maximising
    key s* (nothing when the initial m_0 is the maximum), and the A_final of
    the raw final state at F_T cancels against m_T's own F_T.
"""
import math

import numpy as np


def _log_sigmoid(x):
    return np.where(x >= 0, -np.log1p(np.exp(-np.abs(x))), x - np.log1p(np.exp(-np.abs(x))))


def _sigmoid(x):
    return np.where(x >= 0, 1.0 / (1.0 + np.exp(-np.abs(x))),
                    np.exp(-np.abs(x)) / (1.0 + np.exp(-np.abs(x))))


def _matmul(a, b):
    return a @ b


# The backward's matrix products, by name; ``ops`` may replace any of them
# (e.g. with operands rounded to a tensor-core type) to study precision.
PRODUCTS = ("dP", "G_khat", "G_q", "WS_dnum", "Cprev", "dCb_terms", "dCb_update")


def head_backward(q, k, v, itl, ftl, otl, dh, L, fgate="sigmoid", dC=None, dn=None, ops=None):
    """One head: q, k, v, otl, dh [S, DH]; itl, ftl [S]; dC [DH, DH], dn [DH]
    or None.  Returns dict of gradients dq, dk, dv, di, df, do.  ``ops`` maps
    names in PRODUCTS to replacements for ``a @ b`` in the backward pass."""
    mm = {nm: _matmul for nm in PRODUCTS}
    mm.update(ops or {})
    S, DH = q.shape
    khat = k / math.sqrt(DH)
    log_f = _log_sigmoid(ftl) if fgate == "sigmoid" else ftl.copy()
    o = _sigmoid(otl)
    nch = (S + L - 1) // L
    C = np.zeros((DH, DH))
    n = np.zeros(DH)
    m = 0.0
    saved = []
    num = np.zeros((S, DH))
    nq = np.zeros(S)
    den = np.zeros(S)
    mt = np.zeros(S)
    # ---- forward recompute, chunk by chunk
    for c in range(nch):
        a, e = c * L, min(S, (c + 1) * L)
        b = np.cumsum(log_f[a:e])
        u = itl[a:e] - b
        m_t = np.maximum(b + m, b + np.maximum.accumulate(u))
        causal = np.tril(np.ones((e - a, e - a), dtype=bool))
        W = np.where(causal, np.exp(np.where(causal, b[:, None] - b[None, :] + itl[a:e][None, :]
                                             - m_t[:, None], 0.0)), 0.0)
        Sc = q[a:e] @ khat[a:e].T
        g = np.exp(b + m - m_t)
        num[a:e] = g[:, None] * (q[a:e] @ C.T) + (W * Sc) @ v[a:e]
        nq[a:e] = g * (q[a:e] @ n) + (W * Sc).sum(1)
        den[a:e] = np.maximum(np.abs(nq[a:e]), np.exp(-m_t))
        mt[a:e] = m_t
        m_end = m_t[-1]
        B = b[-1]
        wk = np.exp(B - b + itl[a:e] - m_end)
        saved.append(dict(a=a, e=e, b=b, m_t=m_t, W=W, Sc=Sc, g=g, wk=wk, B=B, m_prev=m,
                          m_end=m_end, C_prev=C.copy(), n_prev=n.copy()))
        decay = np.exp(B + m - m_end)
        C = decay * C + (v[a:e].T * wk) @ khat[a:e]
        n = decay * n + (wk[:, None] * khat[a:e]).sum(0)
        m = m_end
    C_T, n_T = C, n
    ht = num / den[:, None]
    # ---- backward
    dht = dh * o
    d_o = dh * ht * o * (1.0 - o)
    dnum = dht / den[:, None]
    active = np.abs(nq) > np.exp(-mt)
    dnq = np.where(active, -(dht * ht).sum(1) / den * np.sign(nq), 0.0)
    A = (dnum * num).sum(1) + dnq * nq
    dq = np.zeros_like(q)
    dkh = np.zeros_like(q)
    dv = np.zeros_like(q)
    dCb = np.zeros((DH, DH)) if dC is None else dC.copy()
    dnb = np.zeros(DH) if dn is None else dn.copy()
    for sv in reversed(saved):
        a, e = sv["a"], sv["e"]
        W, Sc, g, wk = sv["W"], sv["Sc"], sv["g"], sv["wk"]
        dv[a:e] += wk[:, None] * mm["dCb_terms"](khat[a:e], dCb.T)
        dkh[a:e] += wk[:, None] * (mm["dCb_terms"](v[a:e], dCb) + dnb[None, :])
        dP = mm["dP"](dnum[a:e], v[a:e].T) + dnq[a:e][:, None]
        G = W * dP
        dq[a:e] += mm["G_khat"](G, khat[a:e]) + g[:, None] * (
            mm["Cprev"](dnum[a:e], sv["C_prev"]) + dnq[a:e][:, None] * sv["n_prev"][None, :])
        dkh[a:e] += mm["G_q"](G.T, q[a:e])
        dv[a:e] += mm["WS_dnum"]((W * Sc).T, dnum[a:e])
        decay = np.exp(sv["B"] + sv["m_prev"] - sv["m_end"])
        dCb = decay * dCb + mm["dCb_update"]((dnum[a:e] * g[:, None]).T, q[a:e])
        dnb = decay * dnb + (g * dnq[a:e]) @ q[a:e]
    di = (khat * dkh).sum(1)
    dF = A - di
    if dC is not None or dn is not None:
        A_final = (0.0 if dC is None else float((dC * C_T).sum())) + \
                  (0.0 if dn is None else float((dn * n_T).sum()))
        F = np.cumsum(log_f)
        cand = itl - F
        s_star = int(np.argmax(cand))
        if S and cand[s_star] > 0.0:        # m_0 = 0 is the other candidate
            di[s_star] -= A_final
            dF[s_star] += A_final
    dlogf = np.cumsum(dF[::-1])[::-1]
    df = dlogf * (_sigmoid(-ftl) if fgate == "sigmoid" else 1.0)
    return dict(q=dq, k=dkh / math.sqrt(DH), v=dv, i_pre=di, f_pre=df, o_pre=d_o)


def backward(q, k, v, i_pre, f_pre, o_pre, dh, L, fgate="sigmoid", dC=None, dn=None, ops=None):
    """All heads of [B, NH, S, DH] inputs; returns {name: gradient}."""
    B, NH, S, DH = q.shape
    out = {nm: np.zeros(np.shape(x)) for nm, x in
           (("q", q), ("k", k), ("v", v), ("i_pre", i_pre), ("f_pre", f_pre), ("o_pre", o_pre))}
    for bi in range(B):
        for hi in range(NH):
            g = head_backward(q[bi, hi], k[bi, hi], v[bi, hi], i_pre[bi, hi], f_pre[bi, hi],
                              o_pre[bi, hi], dh[bi, hi], L, fgate,
                              None if dC is None else dC[bi, hi],
                              None if dn is None else dn[bi, hi], ops)
            for nm in out:
                out[nm][bi, hi] = g[nm]
    return out
