"""The mLSTM cell as a differentiable PyTorch op: ``xlstm_mlstm_fwd`` forward,
``xlstm_mlstm_bwd`` backward, through the ctypes binding (argument marshalling
only; every step runs in the library's kernels).

``mlstm_cell(q, k, v, i_pre, f_pre, o_pre)`` returns ``(h, C, n, m)`` for a
zero initial state; h and the final stabilised state (C', n') carry gradients
to q, k, v and the three gate pre-activations.  m, the stabiliser, is
bookkeeping of the stabilised units and is returned without a gradient.
"""
from __future__ import annotations

import torch

from . import binding as xb

BWD_MAX_CHUNK = 64       # the backward kernels hold a chunk of tokens per thread


class MLSTMCellFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, i_pre, f_pre, o_pre, chunk, fgate):
        h, C, n, m = xb.mlstm_fwd(q, k, v, i_pre, f_pre, o_pre, chunk=chunk, fgate=fgate)
        ctx.save_for_backward(q, k, v, i_pre, f_pre, o_pre)
        ctx.chunk = min(chunk, BWD_MAX_CHUNK)
        ctx.fgate = fgate
        ctx.mark_non_differentiable(m)
        return h, C, n, m

    @staticmethod
    def backward(ctx, dh, dC, dn, dm):
        q, k, v, i_pre, f_pre, o_pre = ctx.saved_tensors
        if dh is None:
            dh = torch.zeros_like(q)
        g = xb.mlstm_bwd(q, k, v, i_pre, f_pre, o_pre, dh.to(q.dtype).contiguous(),
                         dC=None if dC is None else dC.float().contiguous(),
                         dn=None if dn is None else dn.float().contiguous(),
                         chunk=ctx.chunk, fgate=ctx.fgate)
        return g["dq"], g["dk"], g["dv"], g["di"], g["df"], g["do"], None, None


def mlstm_cell(q, k, v, i_pre, f_pre, o_pre, chunk=64, fgate="sigmoid"):
    """Differentiable mLSTM cell forward from a zero state: (h, C, n, m)."""
    return MLSTMCellFunction.apply(q, k, v, i_pre, f_pre, o_pre, chunk, fgate)
