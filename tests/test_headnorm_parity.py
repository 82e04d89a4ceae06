"""GPU parity of the block epilogue (``xlstm_mlstm_headnorm_gate``) against the
float64 oracle: per-head GroupNorm, learnable skip and external output gate
("xLSTM: Extended Long Short-Term Memory" section 2.4, Figure 10).

Tolerance, from the arithmetic: the kernel works in fp32 on the same inputs the
oracle sees, so its fp32 result is within a few fp32 roundings of the terms
(mean and variance over <= 512 channels, rsqrt, the gate's exp): below 1e-5 of
max(1, |y|) at these input scales.  A bf16 output adds one rounding to nearest,
at most 2^-8 |y|.  Hence, element by element:
  fp32:  |got - ref| <= 1e-5 * max(1, |ref|)
  bf16:  |got - ref| <= 2^-8 * |ref| + 1e-5 * max(1, max |ref|)
"""
import numpy as np
import pytest
import torch

from oracle.headnorm import headnorm_gate as oracle_headnorm
from linear_rnn_mlstm_b200 import binding as xb
from linear_rnn_mlstm_b200 import synthetic as syn

import parity

pytestmark = pytest.mark.gpu

EPS = 1e-5


def _check(got, ref, dtype, what="y"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    d = np.abs(got - ref)
    if dtype == "bf16":
        bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * max(1.0, float(np.max(np.abs(ref))))
    else:
        bound = 1e-5 * np.maximum(1.0, np.abs(ref))
    worst = int(np.argmax(d - bound))
    assert np.all(d <= bound), (f"{what}: |d| = {d.flat[worst]:.3e} > bound {bound.flat[worst]:.3e} "
                                f"at flat index {worst} (ref {ref.flat[worst]:.6g})")


def _gpu(inp, ogate, eps=EPS):
    d = {k: v.cuda().contiguous() for k, v in inp.items()}
    y = xb.mlstm_headnorm_gate(d["h"], d["gamma"], d["beta"], d["z"], d.get("skip_w"),
                               d.get("x_skip"), eps=eps, ogate=ogate)
    torch.cuda.synchronize()
    assert xb.xlstm_device_status(torch.cuda.current_stream().cuda_stream) == xb.OK
    return y.float().cpu().numpy()


def _ref(inp, ogate, eps=EPS):
    return oracle_headnorm(inp["h"], inp["gamma"], inp["beta"], inp["z"], inp.get("skip_w"),
                           inp.get("x_skip"), eps=eps, ogate=ogate)


# (dtype, DH): every lane-group width the kernel instantiates (2..32 lanes per
# row, and 2 or 4 vectors per lane at DH 512), with B*NH*S = 42 rows: a ragged
# tail for every rows-per-warp count.
CASES = [("bf16", 16, "silu", True), ("bf16", 48, "sigmoid", True), ("bf16", 64, "silu", False),
         ("bf16", 128, "sigmoid", False), ("bf16", 256, "silu", True), ("bf16", 512, "sigmoid", True),
         ("f32", 16, "sigmoid", False), ("f32", 48, "silu", True), ("f32", 128, "silu", True),
         ("f32", 256, "sigmoid", True), ("f32", 512, "silu", False)]


@pytest.mark.parametrize("dtype,DH,ogate,skip", CASES,
                         ids=[f"{c[0]}-DH{c[1]}-{c[2]}-{'skip' if c[3] else 'noskip'}" for c in CASES])
def test_epilogue_matches_oracle(cuda_lib, dtype, DH, ogate, skip):
    inp = syn.epilogue_inputs(2, 3, 7, DH, dtype, seed=DH, skip=skip)
    _check(_gpu(inp, ogate), _ref(inp, ogate), dtype)


# Longer sequences at the wide-row widths (a whole warp per row, one to four
# vectors per lane): row counts that leave every warp of the last pass partly
# empty, with and without the skip input, and fp32 DH 64.
STREAM_CASES = [("bf16", 128, 70, "silu", True), ("bf16", 256, 37, "sigmoid", True),
                ("bf16", 512, 19, "silu", False), ("f32", 64, 70, "sigmoid", True),
                ("f32", 256, 21, "silu", False), ("f32", 512, 10, "sigmoid", True)]


@pytest.mark.parametrize("dtype,DH,S,ogate,skip", STREAM_CASES,
                         ids=[f"{c[0]}-DH{c[1]}-S{c[2]}-{c[3]}-{'skip' if c[4] else 'noskip'}"
                              for c in STREAM_CASES])
def test_epilogue_longer_sequences(cuda_lib, dtype, DH, S, ogate, skip):
    inp = syn.epilogue_inputs(2, 3, S, DH, dtype, seed=DH + S, skip=skip)
    _check(_gpu(inp, ogate), _ref(inp, ogate), dtype)


def test_epilogue_many_rows_grid_stride(cuda_lib):
    """More rows than one resident wave of CTAs: every warp strides."""
    inp = syn.epilogue_inputs(2, 4, 3001, 128, "bf16", seed=5)
    _check(_gpu(inp, "silu"), _ref(inp, "silu"), "bf16")


@pytest.mark.parametrize("DH", [48, 64])
def test_epilogue_constant_rows(cuda_lib, DH):
    """A row with zero variance normalises to zero: y = (beta + skip) * act(z)."""
    inp = syn.epilogue_inputs(1, 2, 5, DH, "bf16", seed=9)
    inp["h"] = torch.full_like(inp["h"], 0.75)
    inp["h"][0, 1, 2] = -3.0
    _check(_gpu(inp, "sigmoid"), _ref(inp, "sigmoid"), "bf16")


def test_epilogue_large_eps_and_single_token(cuda_lib):
    inp = syn.epilogue_inputs(1, 1, 1, 256, "f32", seed=3)
    _check(_gpu(inp, "silu", eps=4.0), _ref(inp, "silu", eps=4.0), "f32")


def test_block_chain_cell_then_epilogue(cuda_lib):
    """The block's form: the cell with its output gate at exactly 1 (otilde =
    +inf, so the gate sits outside the cell), then the epilogue; the CUDA chain
    against the oracle chain, normwise as the cell output is compared."""
    w = syn.custom("chain", 2, 2, 200, 128, syn.SMALL)          # bf16, tensor-core path
    inp = syn.fwd_inputs(w, seed=21)
    inp["o_pre"] = torch.full_like(inp["o_pre"], float("inf"))
    epi = syn.epilogue_inputs(w.B, w.NH, w.S, w.DH, "bf16", seed=22)
    d = parity.to_cuda(inp)
    h, _, _, _ = xb.mlstm_fwd(d["q"], d["k"], d["v"], d["i_pre"], d["f_pre"], d["o_pre"],
                              chunk=64, state_out=False)
    e = {k: v.cuda().contiguous() for k, v in epi.items() if k != "h"}
    y = xb.mlstm_headnorm_gate(h, e["gamma"], e["beta"], e["z"], e["skip_w"], e["x_skip"],
                               eps=EPS, ogate="silu")
    torch.cuda.synchronize()
    assert xb.xlstm_device_status(torch.cuda.current_stream().cuda_stream) == xb.OK
    h_ref = parity.oracle_fwd(inp, w.fgate)[0]
    y_ref = oracle_headnorm(h_ref, epi["gamma"], epi["beta"], epi["z"], epi["skip_w"],
                            epi["x_skip"], eps=EPS, ogate="silu")
    parity.assert_close(h.float().cpu().numpy(), h_ref, "bf16", "cell h")
    parity.assert_close(y.float().cpu().numpy(), y_ref, "bf16", "epilogue y")


def test_epilogue_long_workload_sampled_tokens(cuda_lib):
    """The shape and launch the benchmark times (long workload: B1 NH8 S16384
    DH256, bf16, skip, SiLU): every head of 48 sampled tokens, including the
    first and the last, against the oracle on those tokens."""
    w = syn.LONG
    inp = syn.epilogue_inputs(w.B, w.NH, w.S, w.DH, "bf16", seed=w.seed)
    y = _gpu(inp, "silu")
    toks = np.unique(np.concatenate([[0, w.S - 1],
                                     np.random.default_rng(1).integers(0, w.S, 46)]))
    sub = dict(inp)
    sub["h"] = inp["h"][:, :, toks]
    sub["x_skip"] = inp["x_skip"][:, toks]
    sub["z"] = inp["z"][:, toks]
    _check(y[:, toks], _ref(sub, "silu"), "bf16")
