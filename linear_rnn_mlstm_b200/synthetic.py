"""Seeded synthetic inputs for the mLSTM cell forward and decode step.

This module holds only the workload shapes and the random draws; it contains
none of the cell's arithmetic, so both the CUDA path and the float64 oracle may
use it.  Everything is drawn on the CPU with a ``torch.Generator`` seeded per
workload, in a fixed order (q, k, v, itilde, ftilde, otilde), each tensor as
float32 N(0, 1) mapped affinely to the workload's distribution; q, k, v are
rounded to bfloat16 on the host for bf16 workloads, so the oracle sees exactly
the values the GPU sees.

The distributions follow the pages: keys and values are zero-mean because a
layer norm precedes their projection ("xLSTM: Extended Long Short-Term Memory"
section 2.3), and forget-gate pre-activations are placed around a positive
bias, the long-memory initialisation the section on limitations says must be
chosen with care.  The pages measure on language-modelling data (Wikitext-103
and others) that is neither here nor needed: these synthetic tensors of the
workloads' shapes stand in for it.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    """Shape and gate distributions of one forward workload."""
    name: str
    B: int
    NH: int
    S: int
    DH: int
    dtype: str = "bf16"            # dtype of q, k, v and h: "bf16" or "f32"
    fgate: str = "sigmoid"         # "sigmoid" or "exp"
    i_mu: float = 0.0
    i_sd: float = 1.0
    f_mu: float = 3.0
    f_sd: float = 1.0
    chunks: tuple = (64,)
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.NH * self.S


@dataclass(frozen=True)
class DecodeWorkload:
    """Recurrent decode: a prefill of ``prefill_S`` tokens, then ``steps`` tokens."""
    name: str
    B: int
    NH: int
    DH: int
    steps: int
    prefill_S: int
    prefill_chunk: int = 64
    dtype: str = "bf16"
    fgate: str = "sigmoid"
    i_mu: float = 0.0
    i_sd: float = 1.0
    f_mu: float = 3.0
    f_sd: float = 1.0
    seed: int = 0

    def prefill(self) -> Workload:
        return Workload(self.name + "-prefill", self.B, self.NH, self.prefill_S, self.DH,
                        self.dtype, self.fgate, self.i_mu, self.i_sd, self.f_mu, self.f_sd,
                        (self.prefill_chunk,), self.seed)


# The five workloads: a tiny fp32 case, a small bf16 case, a 1.3B-block-shaped
# case with exponential forget gating and a wide input-gate spread (so the
# stabiliser moves), a long-context case, and the recurrent decode.
TINY = Workload("tiny", 1, 2, 64, 16, "f32", "sigmoid", 0.0, 1.0, 3.0, 1.0, (64,))
SMALL = Workload("small", 4, 4, 1024, 64, "bf16", "sigmoid", 0.0, 1.0, 3.0, 1.0, (64,))
BLOCK = Workload("block", 4, 4, 2048, 512, "bf16", "exp", 0.0, 3.0, -0.05, 0.1, (64, 128))
LONG = Workload("long", 1, 8, 16384, 256, "bf16", "sigmoid", 0.0, 1.0, 4.0, 1.0, (64, 128, 256))
DECODE = DecodeWorkload("decode", 256, 8, 512, 1024, 512)

WORKLOADS = {w.name: w for w in (TINY, SMALL, BLOCK, LONG)}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _qkv_dtype(dtype: str) -> torch.dtype:
    if dtype == "bf16":
        return torch.bfloat16
    if dtype == "f32":
        return torch.float32
    raise ValueError(f"unknown dtype {dtype!r}")


def fwd_inputs(w: Workload, seed: Optional[int] = None, S: Optional[int] = None) -> dict:
    """CPU tensors for one forward: q, k, v [B,NH,S,DH] (workload dtype),
    i_pre, f_pre [B,NH,S] float32, o_pre [B,NH,S,DH] float32."""
    seed = w.seed if seed is None else seed
    S = w.S if S is None else S
    g = _gen(seed)
    shp = (w.B, w.NH, S, w.DH)
    dt = _qkv_dtype(w.dtype)
    q = torch.randn(shp, generator=g, dtype=torch.float32).to(dt)
    k = torch.randn(shp, generator=g, dtype=torch.float32).to(dt)
    v = torch.randn(shp, generator=g, dtype=torch.float32).to(dt)
    i_pre = torch.randn(shp[:3], generator=g, dtype=torch.float32) * w.i_sd + w.i_mu
    f_pre = torch.randn(shp[:3], generator=g, dtype=torch.float32) * w.f_sd + w.f_mu
    o_pre = torch.randn(shp, generator=g, dtype=torch.float32)
    return dict(q=q, k=k, v=v, i_pre=i_pre, f_pre=f_pre, o_pre=o_pre)


def step_inputs(d: DecodeWorkload, step: int, seed: Optional[int] = None) -> dict:
    """CPU tensors for decode token ``step``: q, k, v, o_pre [B,NH,DH],
    i_pre, f_pre [B,NH].  Each step has its own generator, seeded from the
    workload seed and the step index, so any step can be drawn alone."""
    seed = d.seed if seed is None else seed
    g = _gen(1_000_003 * (seed + 1) + 7919 * (step + 1))
    shp = (d.B, d.NH, d.DH)
    dt = _qkv_dtype(d.dtype)
    q = torch.randn(shp, generator=g, dtype=torch.float32).to(dt)
    k = torch.randn(shp, generator=g, dtype=torch.float32).to(dt)
    v = torch.randn(shp, generator=g, dtype=torch.float32).to(dt)
    i_pre = torch.randn(shp[:2], generator=g, dtype=torch.float32) * d.i_sd + d.i_mu
    f_pre = torch.randn(shp[:2], generator=g, dtype=torch.float32) * d.f_sd + d.f_mu
    o_pre = torch.randn(shp, generator=g, dtype=torch.float32)
    return dict(q=q, k=k, v=v, i_pre=i_pre, f_pre=f_pre, o_pre=o_pre)


def custom(name: str, B: int, NH: int, S: int, DH: int, base: Workload = SMALL, **kw) -> Workload:
    """A workload with ``base``'s distributions and the given shape."""
    return replace(base, name=name, B=B, NH=NH, S=S, DH=DH, **kw)


def epilogue_inputs(B: int, NH: int, S: int, DH: int, dtype: str = "bf16", seed: int = 0,
                    skip: bool = True) -> dict:
    """CPU tensors for the block epilogue after the cell (per-head GroupNorm,
    learnable skip, external output gate): h [B,NH,S,DH] and x_skip, z
    [B,S,NH*DH] in ``dtype``; gamma, beta, skip_w [NH*DH] float32.  Scale and
    shift near their identity initialisation; h with a non-zero mean so that
    the centring matters.  Drawn in the order h, gamma, beta, skip_w, x_skip, z."""
    g = _gen(seed)
    dt = _qkv_dtype(dtype)
    D = NH * DH
    h = (torch.randn((B, NH, S, DH), generator=g, dtype=torch.float32) * 1.5 + 0.3).to(dt)
    gamma = torch.randn(D, generator=g, dtype=torch.float32) * 0.1 + 1.0
    beta = torch.randn(D, generator=g, dtype=torch.float32) * 0.1
    skip_w = torch.randn(D, generator=g, dtype=torch.float32) * 0.5
    x_skip = torch.randn((B, S, D), generator=g, dtype=torch.float32).to(dt)
    z = torch.randn((B, S, D), generator=g, dtype=torch.float32).to(dt)
    out = dict(h=h, gamma=gamma, beta=beta, z=z)
    if skip:
        out.update(skip_w=skip_w, x_skip=x_skip)
    return out


# sLSTM timing workload: the 1.3B block width (1024) split over four heads.
SLSTM = dict(B=4, NH=4, S=2048, DH=256)


def slstm_inputs(B: int, NH: int, S: int, DH: int, seed: int = 0) -> dict:
    """CPU float32 tensors for the sLSTM forward: gate pre-activations zx, ix,
    fx, ox [B,NH,S,DH] ~ N(0, 0.5^2) and recurrent blocks R [NH,4,DH,DH] ~
    N(0, 1/DH) per element.  Drawn in the order zx, ix, fx, ox, R."""
    g = _gen(seed)
    shp = (B, NH, S, DH)
    out = {k: torch.randn(shp, generator=g, dtype=torch.float32) * 0.5 for k in ("zx", "ix", "fx", "ox")}
    out["R"] = torch.randn((NH, 4, DH, DH), generator=g, dtype=torch.float32) / DH ** 0.5
    return out
