"""The tensor-core forwards (bf16, chunk 64) against the float64 oracle, forced
through the tensor path, on the cases their design has to get right beyond the
plain workloads.  Two kernel families: the register-state kernel (DH 64, 128,
256; XLSTM_PATH_TENSOR_RS) and the tensor-memory-state kernel (DH 128, 256;
XLSTM_PATH_TENSOR_TMEM); XLSTM_PATH_TENSOR picks between them.  Cases:

- several value-row tiles and several segments per head, ragged tails;
- the exponential forget gate;
- the lazily scaled state: moderate decay, where the state's scale is reset in
  TMEM every few chunks;
- wide chunks: strong decay with large input gates, where one chunk's largest
  input term outweighs the state it starts from by far more than e^60 and the
  exact (unfactorised) intra-chunk weights are used;
- a given initial state folded in before the first chunk;
- configurations the tensor path does not take are refused, not rerouted.
"""
import numpy as np
import pytest
import torch

from linear_rnn_mlstm_b200 import binding as xb
from linear_rnn_mlstm_b200 import synthetic as syn

from parity import STATE_M_ABS, STATE_REL_L2, assert_close, errors, gpu_fwd, oracle_fwd, to_cuda

pytestmark = pytest.mark.gpu


FAMILIES = [xb.PATH_TENSOR_RS, xb.PATH_TENSOR_TMEM]


def _check(inp, fgate, seg, C0=None, n0=None, m0=None, families=FAMILIES, chunk=64):
    hr, Cr, nr, mr = oracle_fwd(inp, fgate, C0, n0, m0)
    DH = inp["q"].shape[-1]
    for fam in families:
        if fam == xb.PATH_TENSOR_TMEM and (DH not in (128, 256) or chunk != 64):
            continue
        h, C, n, m = gpu_fwd(inp, chunk, fgate, fam, seg, C0, n0, m0)
        assert_close(h, hr, "bf16", what=f"h (family {fam})")
        assert errors(C, Cr)[1] <= STATE_REL_L2 and errors(n, nr)[1] <= STATE_REL_L2
        assert np.max(np.abs(m - mr)) <= STATE_M_ABS


CASES = [
    # (B, NH, S, DH, fgate, segments)
    (1, 1, 64, 128, "sigmoid", 0),
    (1, 1, 200, 128, "sigmoid", 0),
    (1, 2, 517, 128, "sigmoid", 1),
    (1, 2, 517, 128, "sigmoid", 4),
    (2, 2, 95, 256, "sigmoid", 0),
    (1, 2, 1000, 256, "exp", 3),
    (1, 1, 1, 128, "sigmoid", 0),
    (1, 1, 63, 256, "exp", 0),
    (2, 1, 640, 256, "sigmoid", 10),
    (1, 1, 64, 64, "sigmoid", 0),
    (1, 2, 300, 512, "exp", 0),
    (2, 1, 517, 512, "sigmoid", 3),
    (2, 3, 777, 64, "sigmoid", 4),
    (1, 2, 300, 64, "exp", 0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_tensor_path_vs_oracle(case):
    B, NH, S, DH, fgate, seg = case
    base = syn.BLOCK if fgate == "exp" else syn.SMALL
    w = syn.custom("tc", B, NH, S, DH, base, dtype="bf16", seed=S + DH)
    _check(syn.fwd_inputs(w), fgate, seg)


@pytest.mark.parametrize("DH", [64, 128, 256, 512])
def test_tensor_path_rescaled_state(DH):
    # log sigmoid(1 +- 0.5) ~ -0.3 per token: the state's scale falls below
    # e^-40 every few chunks and is reset in TMEM
    w = syn.custom("tc_decay", 1, 2, 2000, DH, syn.SMALL, dtype="bf16", seed=7,
                   f_mu=1.0, f_sd=0.5)
    _check(syn.fwd_inputs(w), "sigmoid", 0)


@pytest.mark.parametrize("seg", [0, 3])
@pytest.mark.parametrize("DH", [256, 512])
def test_tensor_path_wide_chunks(seg, DH):
    # log sigmoid(-4 +- 1) ~ -4 per token and itilde ~ N(0, 3): within one chunk
    # the input terms span e^250
    w = syn.custom("tc_wide", 1, 2, 1000, DH, syn.SMALL, dtype="bf16", seed=11,
                   f_mu=-4.0, f_sd=1.0, i_sd=3.0)
    _check(syn.fwd_inputs(w), "sigmoid", seg)


def test_tensor_path_mixed_chunks():
    # wide, rescaled and plain chunks in one sequence: the forget gate drifts
    # from strongly forgetting to remembering over the sequence
    w = syn.custom("tc_mixed", 1, 2, 1536, 128, syn.SMALL, dtype="bf16", seed=5, i_sd=2.0)
    inp = syn.fwd_inputs(w)
    ramp = torch.linspace(-5.0, 6.0, w.S).expand_as(inp["f_pre"])
    inp["f_pre"] = (inp["f_pre"] - w.f_mu) + ramp
    _check(inp, "sigmoid", 2)


def test_tensor_path_initial_state():
    w = syn.custom("tc_init", 2, 2, 300, 128, syn.SMALL, dtype="bf16", seed=3)
    inp = syn.fwd_inputs(w)
    g = torch.Generator().manual_seed(17)
    C0 = torch.randn(2, 2, 128, 128, generator=g) * 0.1
    n0 = torch.randn(2, 2, 128, generator=g) * 0.1
    m0 = torch.randn(2, 2, generator=g)
    for seg in (0, 3):
        _check(inp, "sigmoid", seg, C0, n0, m0)


@pytest.mark.parametrize("dtype,DH,chunk,fam", [("f32", 128, 64, xb.PATH_TENSOR), ("bf16", 48, 64, xb.PATH_TENSOR),
                                                ("bf16", 512, 256, xb.PATH_TENSOR),
                                                ("bf16", 64, 64, xb.PATH_TENSOR_TMEM),
                                                ("bf16", 128, 128, xb.PATH_TENSOR_TMEM)])
def test_tensor_path_refuses_unsupported(dtype, DH, chunk, fam):
    w = syn.custom("tc_unsup", 1, 1, 128, DH, syn.SMALL, dtype=dtype, seed=1)
    d = to_cuda(syn.fwd_inputs(w))
    with pytest.raises(xb.XlstmError) as err:
        xb.mlstm_fwd(d["q"], d["k"], d["v"], d["i_pre"], d["f_pre"], d["o_pre"], chunk=chunk,
                     path=fam)
    assert err.value.status == xb.ERR_UNSUPPORTED


# Chunks of 128 and 256 tokens: the state is carried across chunks only and the
# intra-chunk quadratic form spans the whole chunk (sub-block tiles below the
# diagonal, masked tiles on it); DH 256 at chunk 256 and DH 512 split the key
# columns over two CTAs.
CHUNK_CASES = [
    # (B, NH, S, DH, fgate, segments, chunk)
    (1, 2, 300, 64, "sigmoid", 0, 128),
    (2, 2, 700, 64, "exp", 3, 256),
    (1, 2, 517, 128, "sigmoid", 1, 128),
    (1, 2, 1000, 128, "exp", 3, 256),
    (2, 1, 640, 256, "sigmoid", 0, 128),
    (1, 2, 777, 256, "sigmoid", 2, 256),
    (1, 1, 129, 256, "exp", 0, 256),
    (1, 2, 300, 512, "exp", 0, 128),
    (2, 1, 517, 512, "sigmoid", 3, 128),
]


@pytest.mark.parametrize("case", CHUNK_CASES, ids=lambda c: "x".join(map(str, c)))
def test_tensor_path_long_chunks(case):
    B, NH, S, DH, fgate, seg, chunk = case
    base = syn.BLOCK if fgate == "exp" else syn.SMALL
    w = syn.custom("tc_chunk", B, NH, S, DH, base, dtype="bf16", seed=S + DH + chunk)
    _check(syn.fwd_inputs(w), fgate, seg, chunk=chunk)


@pytest.mark.parametrize("DH,chunk", [(128, 256), (256, 128), (512, 128)])
def test_tensor_path_long_chunks_wide_and_state(DH, chunk):
    # wide chunks (input terms spanning e^250 inside one chunk) and a given
    # initial state, at the longer chunk sizes
    w = syn.custom("tc_chunk_wide", 1, 2, 900, DH, syn.SMALL, dtype="bf16", seed=11 + chunk,
                   f_mu=-4.0, f_sd=1.0, i_sd=3.0)
    _check(syn.fwd_inputs(w), "sigmoid", 0, chunk=chunk)
    w = syn.custom("tc_chunk_init", 2, 2, 300, DH, syn.SMALL, dtype="bf16", seed=3 + chunk)
    g = torch.Generator().manual_seed(17)
    C0 = torch.randn(2, 2, DH, DH, generator=g) * 0.1
    n0 = torch.randn(2, 2, DH, generator=g) * 0.1
    m0 = torch.randn(2, 2, generator=g)
    _check(syn.fwd_inputs(w), "sigmoid", 2, C0, n0, m0, chunk=chunk)
