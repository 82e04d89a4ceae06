"""Sequence-parallel forward: one long sequence split over the ranks of a
process group, each rank holding one contiguous slice of every head.

The mLSTM state after a run of tokens is a fold of per-run summaries
("xLSTM: Extended Long Short-Term Memory" section 2.3, the recurrence unrolled
over a run; the fold is written out in ``include/xlstm_mlstm.h``).  So no rank
waits for its predecessor's forward:

1. every rank but the last summarises its slice from the zero state
   (``xlstm_mlstm_seg_state``: the forward's gate pass and segment summaries,
   no outputs);
2. one all-gather exchanges the summaries (B*NH*(DH*DH + DH + 2) floats per
   rank: 2.1 MB at B1 NH8 DH256);
3. rank r folds the summaries of ranks 0..r-1 onto the initial state
   (``xlstm_mlstm_state_combine``) and runs its slice's forward from there.

Rank r's outputs are exactly the single-sequence forward's outputs for its
slice; the last rank's final state is the sequence's final state.  The
exchange is the only collective.  Every numeric step runs in the library's
kernels; this module moves tensors and calls them.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import binding


class LibraryOps:
    """The library's entry points (the default; CUDA tensors)."""
    dtype = torch.float32

    @staticmethod
    def floats(B, NH, DH):
        return binding.seg_state_floats(B, NH, DH)

    @staticmethod
    def seg_state(k, v, i_pre, f_pre, chunk, fgate):
        return binding.mlstm_seg_state(k, v, i_pre, f_pre, chunk=chunk, fgate=fgate)

    @staticmethod
    def combine(parts, count, B, NH, DH, C0, n0, m0):
        return binding.mlstm_state_combine(parts, count, B, NH, DH, C0=C0, n0=n0, m0=m0)

    @staticmethod
    def fwd(q, k, v, i_pre, f_pre, o_pre, chunk, fgate, C0, n0, m0):
        return binding.mlstm_fwd(q, k, v, i_pre, f_pre, o_pre, chunk=chunk, fgate=fgate, C0=C0,
                                 n0=n0, m0=m0)


def _all_gather(packed: torch.Tensor, world: int, group) -> torch.Tensor:
    out = torch.empty((world, packed.numel()), dtype=packed.dtype, device=packed.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, packed, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), packed, group=group)
    return out


def sequence_parallel_fwd(q, k, v, i_pre, f_pre, o_pre, chunk: int = 64, fgate: str = "sigmoid",
                          C0=None, n0=None, m0=None, group=None, ops=None,
                          timings: Optional[dict] = None):
    """Forward of this rank's slice of a sequence split over ``group``.

    q, k, v, o_pre [B, NH, S_r, DH], i_pre, f_pre [B, NH, S_r]: this rank's
    slice (S_r may differ between ranks; ranks are in sequence order).
    (C0, n0, m0): the sequence's initial state (the same on every rank; None =
    zero).  Returns (h, C, n, m): h of the slice and the state at the slice's
    end.  ``timings`` (optional dict) receives CUDA events around the phases
    when the tensors are on a GPU.
    """
    ops = LibraryOps() if ops is None else ops
    distributed = dist.is_available() and dist.is_initialized()
    world = dist.get_world_size(group) if distributed else 1
    rank = dist.get_rank(group) if distributed else 0
    if world == 1:
        return ops.fwd(q, k, v, i_pre, f_pre, o_pre, chunk, fgate, C0, n0, m0)
    B, NH, S, DH = q.shape
    nf = ops.floats(B, NH, DH)
    ev = (lambda: torch.cuda.Event(enable_timing=True)) if q.is_cuda and timings is not None else None
    marks = [ev()] if ev else []
    if marks:
        marks[0].record()
    if rank < world - 1:
        packed = ops.seg_state(k, v, i_pre, f_pre, chunk, fgate)
    else:
        # the last slice's summary is folded by nobody: its slot is never read
        packed = torch.empty(nf, dtype=getattr(ops, "dtype", torch.float32), device=q.device)
    if ev:
        marks.append(ev())
        marks[-1].record()
    parts = _all_gather(packed, world, group)
    if ev:
        marks.append(ev())
        marks[-1].record()
    if rank == 0:
        Cs, ns, ms = C0, n0, m0
    else:
        Cs, ns, ms = ops.combine(parts, rank, B, NH, DH, C0, n0, m0)
    out = ops.fwd(q, k, v, i_pre, f_pre, o_pre, chunk, fgate, Cs, ns, ms)
    if ev:
        marks.append(ev())
        marks[-1].record()
        timings["events"] = marks       # seg_state | exchange | combine + forward
    return out
