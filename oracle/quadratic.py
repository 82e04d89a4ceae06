"""Quadratic (parallel) form of the mLSTM cell, float64, for tiny inputs.

"xLSTM: Extended Long Short-Term Memory" section 2.3 states that, because
mLSTM has no memory mixing, its recurrence can be rewritten in a parallel form
(its appendix A.3, which the pages do not reproduce).  This module derives
that form by unrolling the raw recurrence from a zero state:

    C_t = sum_{s<=t} (prod_{j=s+1..t} f_j) i_s v_s khat_s^T
        = sum_{s<=t} exp(F_t - F_s + itilde_s) v_s khat_s^T,   F_t = sum_{j<=t} log f_j

so that, with D_ts = exp(F_t - F_s + itilde_s) for s <= t and 0 otherwise,

    h_t = sigmoid(otilde_t) * sum_s D_ts (q_t . khat_s) v_s
                              / max(|sum_s D_ts (q_t . khat_s)|, 1).

Nothing here is shared with the C recurrence in ``mlstm_oracle.c``: the gate
activations are written differently (numpy's logaddexp for log sigmoid), no
stabiliser is used, and the sums run in matrix form.  It is test
infrastructure: the tests compare it with the recurrence on tiny inputs.
"""
from __future__ import annotations

import numpy as np


def _np(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def quadratic_form(q, k, v, i_pre, f_pre, o_pre, fgate="sigmoid"):
    """h [B, NH, S, DH] from the explicit decay matrix D (zero initial state)."""
    q, k, v, o_pre = _np(q), _np(k), _np(v), _np(o_pre)
    i_pre, f_pre = _np(i_pre), _np(f_pre)
    B, NH, S, DH = q.shape
    if fgate == "exp":
        log_f = f_pre
    else:
        log_f = -np.logaddexp(0.0, -f_pre)          # log(1 / (1 + e^-x))
    F = np.cumsum(log_f, axis=-1)                    # [B, NH, S]
    log_D = F[..., :, None] - F[..., None, :] + i_pre[..., None, :]
    causal = np.tril(np.ones((S, S), dtype=bool))
    D = np.where(causal, np.exp(np.where(causal, log_D, 0.0)), 0.0)
    khat = k / np.sqrt(DH)
    scores = np.einsum("bhtd,bhsd->bhts", q, khat)
    W = D * scores
    num = np.einsum("bhts,bhsd->bhtd", W, v)
    den = np.abs(W.sum(axis=-1))
    with np.errstate(over="ignore"):
        o = 1.0 / (1.0 + np.exp(-o_pre))
    return o * num / np.maximum(den, 1.0)[..., None]
