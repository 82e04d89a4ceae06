"""GPU parity of the sequence-parallel calls against the oracle.

xlstm_mlstm_seg_state must give the slice summary the oracle gives (the
recurrence from the zero state with stabiliser -inf, and the slice's total
log forget); xlstm_mlstm_state_combine must give the state the oracle reaches
after the prefix of slices; and ranks emulated one after another on this GPU
(summaries, the gathered array, the fold, each slice's forward from its
folded state) must reproduce the single-sequence oracle's h and final state.
The same calls run one per GPU under ``seqpar.sequence_parallel_fwd``; its
collective plumbing is covered on gloo ranks in test_seqpar.py."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_mlstm_b200 import binding as xb
from linear_rnn_mlstm_b200 import synthetic as syn

from parity import STATE_M_ABS, STATE_REL_L2, assert_close, errors, fp32_arith, to_cuda

pytestmark = pytest.mark.gpu

KEYS = ("q", "k", "v", "i_pre", "f_pre", "o_pre")

# (workload base, B, NH, S, DH, qkv dtype, chunk): the tensor-core summaries at
# every DH they take (the tensor-memory kernel's DH 128 / 256 with chunk 64, the
# register-state family's DH 64 / 512 and chunk 128 / 256), ragged S, and the
# fp32 kernels.
CASES = [
    ("small-dh64", syn.SMALL, 2, 2, 333, 64, "bf16", 64),
    ("long-dh128", syn.LONG, 1, 2, 1000, 128, "bf16", 64),
    ("long-dh256-L128", syn.LONG, 1, 2, 700, 256, "bf16", 128),
    ("long-dh256-L256", syn.LONG, 1, 1, 1300, 256, "bf16", 256),
    ("block-dh512", syn.BLOCK, 1, 2, 300, 512, "bf16", 64),
    ("small-dh48-simt", syn.SMALL, 1, 2, 150, 48, "bf16", 64),
    ("tiny-f32", syn.TINY, 1, 2, 77, 32, "f32", 16),
]


def _inputs(base, B, NH, S, DH, dtype, seed=7):
    return syn.fwd_inputs(syn.custom("sp", B, NH, S, DH, base, dtype=dtype), seed=seed)


def _slice(inp, a, b):
    return {k: v[:, :, a:b].contiguous() for k, v in inp.items()}


def _log_forget(f_pre, fgate):
    f = np.asarray(f_pre, dtype=np.float64)
    return f if fgate == "exp" else -np.logaddexp(0.0, -f)


def _oracle_summary(inp, fgate):
    B, NH, S, DH = inp["k"].shape
    zeros = np.zeros((B, NH, S, DH))
    _, C, n, m = oracle.fwd(zeros, inp["k"], inp["v"], inp["i_pre"], inp["f_pre"], zeros, fgate,
                            None, None, np.full((B, NH), -np.inf))
    return C, n, m, _log_forget(inp["f_pre"], fgate).sum(axis=-1)


def _state_tol(dtype, DH, chunk):
    # fp32-arithmetic summaries are held like the fp32 forward's state
    return 1e-5 if dtype == "f32" or fp32_arith(DH, chunk, dtype) else STATE_REL_L2


def _check_state(got, ref, tol):
    C, n, m = got
    Cr, nr, mr = ref
    assert errors(C, Cr)[1] <= tol, errors(C, Cr)
    assert errors(n, nr)[1] <= tol, errors(n, nr)
    assert np.max(np.abs(np.asarray(m, dtype=np.float64) - mr)) <= STATE_M_ABS


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_seg_state_matches_oracle(case):
    _, base, B, NH, S, DH, dtype, chunk = case
    inp = _inputs(base, B, NH, S, DH, dtype)
    d = to_cuda(inp)
    packed = xb.mlstm_seg_state(d["k"], d["v"], d["i_pre"], d["f_pre"], chunk=chunk, fgate=base.fgate)
    torch.cuda.synchronize()
    assert xb.xlstm_device_status(torch.cuda.current_stream().cuda_stream) == xb.OK
    C, n, m, F = (t.cpu().numpy() for t in xb.unpack_seg_state(packed, B, NH, DH))
    Cr, nr, mr, Fr = _oracle_summary(inp, base.fgate)
    _check_state((C, n, m), (Cr, nr, mr), _state_tol(dtype, DH, chunk))
    np.testing.assert_allclose(F, Fr, rtol=1e-5, atol=1e-4)


def test_seg_state_of_an_empty_slice_is_the_identity():
    packed = torch.full((xb.seg_state_floats(1, 2, 64),), 7.0, device="cuda")
    e = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device="cuda")
    g = torch.empty((1, 2, 0), dtype=torch.float32, device="cuda")
    xb.mlstm_seg_state(e, e, g, g, packed=packed)
    C, n, m, F = (t.cpu().numpy() for t in xb.unpack_seg_state(packed, 1, 2, 64))
    assert not C.any() and not n.any() and not F.any() and np.all(m == -np.inf)


def _emulate_ranks(inp, bounds, chunk, fgate, init):
    """Every rank's calls, one after another on this GPU; returns each slice's
    (h, C, n, m) and the folded incoming states."""
    B, NH, S, DH = inp["q"].shape
    R = len(bounds) - 1
    sl = [to_cuda(_slice(inp, a, b)) for a, b in zip(bounds[:-1], bounds[1:])]
    nf = xb.seg_state_floats(B, NH, DH)
    parts = torch.zeros((R, nf), dtype=torch.float32, device="cuda")
    for r in range(R - 1):
        xb.mlstm_seg_state(sl[r]["k"], sl[r]["v"], sl[r]["i_pre"], sl[r]["f_pre"], chunk=chunk,
                           fgate=fgate, packed=parts[r])
    C0, n0, m0 = (None if t is None else torch.as_tensor(t, dtype=torch.float32).cuda() for t in init)
    outs, incoming = [], []
    for r in range(R):
        if r == 0:
            st = (C0, n0, m0)
        else:
            st = xb.mlstm_state_combine(parts, r, B, NH, DH, C0=C0, n0=n0, m0=m0)
        incoming.append(st)
        outs.append(xb.mlstm_fwd(*(sl[r][k] for k in KEYS), chunk=chunk, fgate=fgate, C0=st[0], n0=st[1],
                                 m0=st[2]))
    torch.cuda.synchronize()
    assert xb.xlstm_device_status(torch.cuda.current_stream().cuda_stream) == xb.OK
    return outs, incoming


@pytest.mark.parametrize("case,bounds", [
    (CASES[0], (0, 100, 200, 333)),
    (CASES[1], (0, 256, 640, 1000)),
    (CASES[2], (0, 300, 301, 700)),
    (CASES[4], (0, 128, 300)),
    (CASES[5], (0, 50, 50, 150)),
    (CASES[6], (0, 20, 41, 60, 77)),
], ids=["small-dh64", "long-dh128", "long-dh256-L128", "block-dh512", "simt-empty-slice", "tiny-f32"])
@pytest.mark.parametrize("with_init", [False, True])
def test_emulated_ranks_reproduce_the_single_sequence_forward(case, bounds, with_init):
    _, base, B, NH, S, DH, dtype, chunk = case
    inp = _inputs(base, B, NH, S, DH, dtype)
    init = (None, None, None)
    if with_init:
        g = np.random.default_rng(9)
        init = (0.1 * g.normal(size=(B, NH, DH, DH)), 0.1 * g.normal(size=(B, NH, DH)),
                g.normal(size=(B, NH)))
    outs, incoming = _emulate_ranks(inp, bounds, chunk, base.fgate, init)
    h = np.concatenate([o[0].float().cpu().numpy() for o in outs], axis=2)
    hr, Cr, nr, mr = oracle.fwd(*(inp[k] for k in KEYS), base.fgate, *init)
    tol = "f32" if dtype == "f32" else "bf16"
    assert_close(h, hr, tol, elementwise=dtype == "f32" or fp32_arith(DH, chunk, dtype))
    st_tol = _state_tol(dtype, DH, chunk)
    _check_state([t.cpu().numpy() for t in outs[-1][1:]], (Cr, nr, mr), st_tol)
    for r in range(1, len(bounds) - 1):
        # the folded incoming state of slice r is the oracle's state after slices 0..r-1
        if bounds[r] == 0:
            continue
        _, *ref = oracle.fwd(*(_slice(inp, 0, bounds[r])[k] for k in KEYS), base.fgate, *init)
        _check_state([t.cpu().numpy() for t in incoming[r]], ref, st_tol)


def test_long_workload_split_over_eight_ranks():
    """The long-context workload's shape (S 16384, DH 256, chunk 64; two of its
    eight heads) cut into eight 2048-token slices."""
    w = syn.LONG
    inp = _inputs(w, 1, 2, w.S, w.DH, "bf16", seed=w.seed)
    bounds = tuple(range(0, w.S + 1, w.S // 8))
    outs, _ = _emulate_ranks(inp, bounds, 64, w.fgate, (None, None, None))
    h = np.concatenate([o[0].float().cpu().numpy() for o in outs], axis=2)
    hr, Cr, nr, mr = oracle.fwd(*(inp[k] for k in KEYS), w.fgate)
    assert_close(h, hr, "bf16")
    _check_state([t.cpu().numpy() for t in outs[-1][1:]], (Cr, nr, mr), STATE_REL_L2)
