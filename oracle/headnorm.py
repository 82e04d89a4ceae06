"""Per-head GroupNorm, learnable skip and external output gate of the mLSTM
block, float64 numpy (test infrastructure only: only ``tests/``, the smoke
entry point and the CPU-baseline leg of the benchmark may import it).

"xLSTM: Extended Long Short-Term Memory" section 2.4, Figure 10 (the mLSTM
block with pre up-projection): the cell's output is normalised by a GroupNorm
whose groups are the heads -- a LayerNorm per head -- then the learnable skip
input is added, and the sum is gated component-wise by the block's external
output gate; a down-projection follows (not part of this op).

GroupNorm (Wu & He, 2018), per sample and group: mean and biased variance over
the group's channels, (x - mean) / sqrt(var + eps), then a per-channel scale
gamma and shift beta.  Here a "sample" is one token of one batch row and the
groups are the NH heads of DH channels each, channel c = head * DH + j.

The pages leave two things open; the readings taken here:
  * the learnable skip is a per-channel weight times the skip input (the cell
    input after the causal convolution), added after the normalisation;
  * the external gate's activation is not named for the mLSTM block; the
    block's activation is Swish (SiLU, z * sigmoid(z)), the default here, and
    the logistic sigmoid of the cell's own output gate is the alternative.

Layouts: h [B, NH, S, DH] (the cell's layout), gamma / beta / skip_w [NH*DH],
x_skip / z / y [B, S, NH*DH] (the block's layout, heads concatenated along the
feature axis).
"""
from __future__ import annotations

import numpy as np

OGATES = ("silu", "sigmoid")


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (any dtype) -> exact float64 copy
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def gate(z, ogate="silu"):
    """The external output gate's activation, elementwise."""
    z = _f64(z)
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-z))
    if ogate == "sigmoid":
        return sig
    if ogate == "silu":
        return z * sig
    raise ValueError(f"ogate must be one of {OGATES}")


def headnorm_gate(h, gamma, beta, z, skip_w=None, x_skip=None, eps=1e-5, ogate="silu"):
    """y = (GroupNorm_heads(h) * gamma + beta + skip_w * x_skip) * gate(z).

    Returns y [B, S, NH*DH] as float64.  ``skip_w`` and ``x_skip`` are both
    given or both omitted (no skip term)."""
    h = _f64(h)
    if h.ndim != 4:
        raise ValueError("h must be [B, NH, S, DH]")
    if (skip_w is None) != (x_skip is None):
        raise ValueError("skip_w and x_skip go together")
    if not eps > 0:
        raise ValueError("eps must be positive")
    B, NH, S, DH = h.shape
    # the cell's [B, NH, S, DH] as tokens x heads x channels-of-a-head
    x = h.transpose(0, 2, 1, 3)
    mean = x.mean(axis=3, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=3, keepdims=True)
    xn = (x - mean) / np.sqrt(var + eps)
    y = xn.reshape(B, S, NH * DH) * _f64(gamma) + _f64(beta)
    if skip_w is not None:
        y = y + _f64(skip_w) * _f64(x_skip).reshape(B, S, NH * DH)
    return y * gate(_f64(z).reshape(B, S, NH * DH), ogate)
