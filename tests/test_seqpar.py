"""Sequence parallelism on the CPU.

1. The fold that joins slice summaries (written out in include/xlstm_mlstm.h,
   from the recurrence of "xLSTM: Extended Long Short-Term Memory" section 2.3
   unrolled over a slice) is pinned to the oracle: slice summaries taken by the
   oracle itself (zero state, stabiliser -inf) and folded in float64 must give
   the state the oracle reaches running the whole prefix token by token.
2. The orchestration in ``seqpar.sequence_parallel_fwd`` (who summarises, the
   all-gather, which prefix each rank folds, the forward from the folded
   state) runs on 2 and 3 gloo ranks with oracle-backed stand-ins for the
   library calls; every rank's h and end state must equal the single-sequence
   oracle's on its slice.
The library's own kernels are held to the same oracle on the GPU
(test_zzz_seqpar_parity.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from linear_rnn_mlstm_b200 import synthetic as syn


def _log_forget(f_pre, fgate):
    f = np.asarray(f_pre, dtype=np.float64)
    return f if fgate == "exp" else -np.logaddexp(0.0, -f)


def _summary(inp, fgate):
    """(C', n', mloc, F) of one slice from the zero state, by the oracle."""
    B, NH, S, DH = inp["k"].shape
    zeros = np.zeros((B, NH, S, DH))
    _, C, n, m = oracle.fwd(zeros, inp["k"], inp["v"], inp["i_pre"], inp["f_pre"], zeros, fgate,
                            None, None, np.full((B, NH), -np.inf))
    F = _log_forget(inp["f_pre"], fgate).sum(axis=-1)
    return C, n, m, F


def _fold(parts, C0=None, n0=None, m0=None, shape=None):
    """The fold of the header, in float64 (the stand-in for the combine kernel)."""
    B, NH, DH = shape
    C = np.zeros((B, NH, DH, DH)) if C0 is None else np.asarray(C0, dtype=np.float64).copy()
    n = np.zeros((B, NH, DH)) if n0 is None else np.asarray(n0, dtype=np.float64).copy()
    M = np.zeros((B, NH)) if m0 is None else np.asarray(m0, dtype=np.float64).copy()
    for Cj, nj, mj, Fj in parts:
        Mn = np.maximum(Fj + M, mj)
        with np.errstate(invalid="ignore"):
            al = np.where(Mn == -np.inf, 0.0, np.exp(Fj + M - Mn))
            be = np.where(Mn == -np.inf, 0.0, np.exp(mj - Mn))
        C = al[..., None, None] * C + be[..., None, None] * Cj
        n = al[..., None] * n + be[..., None] * nj
        M = Mn
    return C, n, M


def _slice(inp, a, b):
    return {k: v[:, :, a:b] for k, v in inp.items()}


@pytest.mark.parametrize("fgate,base", [("sigmoid", syn.SMALL), ("exp", syn.BLOCK)])
@pytest.mark.parametrize("bounds", [(0, 9, 20, 33), (0, 1, 2, 40), (0, 17, 17, 30)])
@pytest.mark.parametrize("with_init", [False, True])
def test_fold_of_oracle_summaries_is_the_recurrence(fgate, base, bounds, with_init):
    w = syn.custom("sp", 2, 2, bounds[-1], 8, base, dtype="f32")
    inp = syn.fwd_inputs(w, seed=3)
    B, NH, DH = 2, 2, 8
    init = (None, None, None)
    if with_init:
        g = np.random.default_rng(5)
        init = (g.normal(size=(B, NH, DH, DH)), g.normal(size=(B, NH, DH)), g.normal(size=(B, NH)))
    parts = [_summary(_slice(inp, a, b), fgate) for a, b in zip(bounds[:-1], bounds[1:])]
    for r in range(len(parts) + 1):
        C, n, M = _fold(parts[:r], *init, shape=(B, NH, DH))
        end = bounds[r]
        if end == 0:
            ref = [np.zeros((B, NH, DH, DH)) if init[0] is None else init[0],
                   np.zeros((B, NH, DH)) if init[1] is None else init[1],
                   np.zeros((B, NH)) if init[2] is None else init[2]]
        else:
            _, *ref = oracle.fwd(*(_slice(inp, 0, end)[k] for k in ("q", "k", "v", "i_pre", "f_pre", "o_pre")),
                                 fgate, *init)
        np.testing.assert_allclose(M, ref[2], rtol=0, atol=1e-12)
        np.testing.assert_allclose(C, ref[0], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(n, ref[1], rtol=1e-10, atol=1e-12)


def test_empty_slice_is_the_identity_of_the_fold():
    w = syn.custom("sp", 1, 2, 12, 8, syn.SMALL, dtype="f32")
    inp = syn.fwd_inputs(w, seed=1)
    empty = (np.zeros((1, 2, 8, 8)), np.zeros((1, 2, 8)), np.full((1, 2), -np.inf), np.zeros((1, 2)))
    full = _summary(inp, "sigmoid")
    for parts in ([empty, full], [full, empty], [empty, empty, full, empty]):
        C, n, M = _fold(parts, shape=(1, 2, 8))
        C1, n1, M1 = _fold([full], shape=(1, 2, 8))
        np.testing.assert_allclose(C, C1, rtol=1e-14, atol=0)
        np.testing.assert_allclose(M, M1, rtol=0, atol=0)


# ------------------------------------------------------------ gloo ranks
class OracleOps:
    """Stand-ins for the library calls (float64, CPU tensors)."""
    dtype = torch.float64

    @staticmethod
    def floats(B, NH, DH):
        n = B * NH * (DH * DH + DH + 2)
        return (n + 3) // 4 * 4

    @staticmethod
    def seg_state(k, v, i_pre, f_pre, chunk, fgate):
        inp = dict(k=k, v=v, i_pre=i_pre, f_pre=f_pre)
        B, NH, S, DH = k.shape
        parts = [np.asarray(x, dtype=np.float64).ravel() for x in _summary(inp, fgate)]
        flat = np.concatenate(parts)
        out = np.zeros(OracleOps.floats(B, NH, DH))
        out[:flat.size] = flat
        return torch.from_numpy(out)

    @staticmethod
    def combine(parts, count, B, NH, DH, C0, n0, m0):
        BH = B * NH
        o1, o2 = BH * DH * DH, BH * DH * DH + BH * DH
        unpacked = []
        for r in range(count):
            p = parts[r].numpy()
            unpacked.append((p[:o1].reshape(B, NH, DH, DH), p[o1:o2].reshape(B, NH, DH),
                             p[o2:o2 + BH].reshape(B, NH), p[o2 + BH:o2 + 2 * BH].reshape(B, NH)))
        return _fold(unpacked, C0, n0, m0, shape=(B, NH, DH))

    @staticmethod
    def fwd(q, k, v, i_pre, f_pre, o_pre, chunk, fgate, C0, n0, m0):
        return oracle.fwd(q, k, v, i_pre, f_pre, o_pre, fgate, C0, n0, m0)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, bounds, fgate, with_init, out):
    from linear_rnn_mlstm_b200 import replicas, seqpar
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    e = replicas.rank_env()
    replicas.init(e, "gloo", timeout_s=60)
    try:
        base = syn.BLOCK if fgate == "exp" else syn.SMALL
        w = syn.custom("sp", 1, 3, bounds[-1], 8, base, dtype="f32")
        inp = syn.fwd_inputs(w, seed=11)
        init = (None, None, None)
        if with_init:
            g = np.random.default_rng(2)
            init = (g.normal(size=(1, 3, 8, 8)), g.normal(size=(1, 3, 8)), g.normal(size=(1, 3)))
        mine = _slice(inp, bounds[rank], bounds[rank + 1])
        h, C, n, m = seqpar.sequence_parallel_fwd(
            *(mine[k] for k in ("q", "k", "v", "i_pre", "f_pre", "o_pre")), chunk=4, fgate=fgate,
            C0=init[0], n0=init[1], m0=init[2], ops=OracleOps())
        ref_h, *_ = oracle.fwd(*(inp[k] for k in ("q", "k", "v", "i_pre", "f_pre", "o_pre")), fgate, *init)
        _, *ref_state = oracle.fwd(*(_slice(inp, 0, bounds[rank + 1])[k]
                                     for k in ("q", "k", "v", "i_pre", "f_pre", "o_pre")), fgate, *init)
        dh = float(np.max(np.abs(h - ref_h[:, :, bounds[rank]:bounds[rank + 1]]), initial=0.0))
        ds = max(float(np.max(np.abs(a - b))) for a, b in zip((C, n, m), ref_state))
        out[rank] = (dh, ds)
        replicas.barrier(e)
    finally:
        replicas.shutdown(e)


@pytest.mark.parametrize("bounds,fgate,with_init", [
    ((0, 13, 29), "sigmoid", False),
    ((0, 8, 19, 31), "exp", True),
    ((0, 10, 10, 24), "sigmoid", True),      # an empty slice in the middle
])
def test_gloo_ranks_reproduce_the_single_sequence_forward(bounds, fgate, with_init):
    world, port = len(bounds) - 1, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, bounds, fgate, with_init, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    for r in range(world):
        dh, ds = out[r]
        assert dh <= 1e-10 and ds <= 1e-10, (r, dh, ds)


def test_one_process_is_the_plain_forward():
    from linear_rnn_mlstm_b200 import seqpar
    w = syn.custom("sp", 1, 2, 20, 8, syn.SMALL, dtype="f32")
    inp = syn.fwd_inputs(w, seed=4)
    args = [inp[k] for k in ("q", "k", "v", "i_pre", "f_pre", "o_pre")]
    h, C, n, m = seqpar.sequence_parallel_fwd(*args, chunk=4, ops=OracleOps())
    ref = oracle.fwd(*args, "sigmoid")
    for a, b in zip((h, C, n, m), ref):
        np.testing.assert_array_equal(a, b)
