"""Gradients of the mLSTM cell, float64 on the CPU (test infrastructure only:
only ``tests/``, the smoke entry point and the CPU-baseline leg of the
benchmark may import it).

The gradient of a loss through the cell has a plain definition: the derivative
of the forward.  This module writes the forward out once more, as the
sequential recurrence of "xLSTM: Extended Long Short-Term Memory" section 2.3
(matrix memory, covariance rule eq. (18), normaliser floored at 1.0) with the
stabiliser of section 2.2, one token at a time in plain PyTorch float64 ops,
and lets PyTorch's reverse-mode differentiation take the derivative -- no
blocking, no chunking, no hand-derived backward.  Section 2.2 (and its
appendix A.2) claims that the stabilised gates f', i' change neither the
output nor the derivatives of the loss; ``raw=True`` differentiates the
unstabilised recurrence so that the tests can check that claim.

The loss is L = sum(dh * h) + sum(dC * C'_T) + sum(dn * n'_T), i.e. the
cotangents dh of the output and, optionally, dC, dn of the final stabilised
state (what a chunked training step passes back into the cell); the returned
gradients are dL/dq, dL/dk, dL/dv, dL/d(itilde), dL/d(ftilde), dL/d(otilde).

Shapes as for the forward: q, k, v, o_pre, dh [B, NH, S, DH]; i_pre, f_pre
[B, NH, S]; dC [B, NH, DH, DH] (row = value index); dn [B, NH, DH].
"""
from __future__ import annotations

import math

import numpy as np
import torch

GRAD_NAMES = ("q", "k", "v", "i_pre", "f_pre", "o_pre")


def _t(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).clone()
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def forward(q, k, v, i_pre, f_pre, o_pre, fgate="sigmoid", raw=False):
    """The recurrence on float64 torch tensors (differentiable).  Returns h and
    the final state (C, n) in stabilised units (raw units when ``raw``)."""
    B, NH, S, DH = q.shape
    khat = k / math.sqrt(DH)
    if fgate == "sigmoid":
        log_f = torch.nn.functional.logsigmoid(f_pre)
    elif fgate == "exp":
        log_f = f_pre
    else:
        raise ValueError("fgate must be 'sigmoid' or 'exp'")
    log_i = i_pre
    o = torch.sigmoid(o_pre)
    C = torch.zeros((B, NH, DH, DH), dtype=torch.float64)
    n = torch.zeros((B, NH, DH), dtype=torch.float64)
    m = torch.zeros((B, NH), dtype=torch.float64)
    hs = []
    for t in range(S):
        kt, vt, qt = khat[:, :, t], v[:, :, t], q[:, :, t]
        if raw:
            fg = torch.exp(log_f[:, :, t])
            ig = torch.exp(log_i[:, :, t])
            floor = torch.ones((B, NH), dtype=torch.float64)
        else:
            m_new = torch.maximum(log_f[:, :, t] + m, log_i[:, :, t])
            fg = torch.exp(log_f[:, :, t] + m - m_new)
            ig = torch.exp(log_i[:, :, t] - m_new)
            floor = torch.exp(-m_new)
            m = m_new
        C = fg[..., None, None] * C + ig[..., None, None] * (vt[..., :, None] * kt[..., None, :])
        n = fg[..., None] * n + ig[..., None] * kt
        num = (C * qt[..., None, :]).sum(-1)
        den = torch.maximum(torch.abs((n * qt).sum(-1)), floor)
        hs.append(o[:, :, t] * num / den[..., None])
    h = torch.stack(hs, dim=2) if S else torch.zeros((B, NH, 0, DH), dtype=torch.float64)
    return h, C, n


def grads(q, k, v, i_pre, f_pre, o_pre, dh, fgate="sigmoid", dC=None, dn=None, raw=False):
    """dL/d(input) for L = sum(dh h) + sum(dC C_T) + sum(dn n_T).  Returns
    (L, {name: float64 numpy array}) with names ``GRAD_NAMES``."""
    # the caller may be inside torch.no_grad() (e.g. an autograd backward):
    # the derivative is taken here regardless
    with torch.enable_grad():
        xs = {nm: _t(x).requires_grad_(True) for nm, x in
              zip(GRAD_NAMES, (q, k, v, i_pre, f_pre, o_pre))}
        h, C, n = forward(*(xs[nm] for nm in GRAD_NAMES), fgate=fgate, raw=raw)
        loss = (h * _t(dh)).sum()
        if dC is not None:
            loss = loss + (C * _t(dC)).sum()
        if dn is not None:
            loss = loss + (n * _t(dn)).sum()
        if loss.requires_grad:
            loss.backward()
    # an input the loss does not reach (e.g. every input of an empty sequence)
    # has a zero gradient
    return float(loss.detach()), {nm: (xs[nm].grad.numpy().copy() if xs[nm].grad is not None
                                       else np.zeros(tuple(xs[nm].shape))) for nm in GRAD_NAMES}
