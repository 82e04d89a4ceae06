"""GPU forward vs the float64 oracle, element by element, on seeded inputs.

Covers the five workload shapes at full size (the decode workload's prefill is
covered in test_step_parity.py), ragged sequence tails (S not a multiple of the
chunk), several value-row tiles, several sequence segments per head (the
two-level chunk-state scan), a given initial state, and the degenerate sizes.
"""
import numpy as np
import pytest
import torch

from linear_rnn_mlstm_b200 import binding as xb
from linear_rnn_mlstm_b200 import synthetic as syn

from parity import (STATE_M_ABS, STATE_REL_L2, assert_close, errors, fp32_arith, gpu_fwd,
                    oracle_fwd)

pytestmark = pytest.mark.gpu

_oracle_cache = {}


def _oracle(w, inp):
    key = (w, id(inp))
    if key not in _oracle_cache:
        _oracle_cache[key] = oracle_fwd(inp, w.fgate)
    return _oracle_cache[key]


_input_cache = {}


def _inputs(w):
    if w not in _input_cache:
        _input_cache[w] = syn.fwd_inputs(w)
    return _input_cache[w]


def _check_state(C, n, m, Cr, nr, mr, dtype):
    if dtype in ("f32", "f32_wide"):
        tol = 1e-5 if dtype == "f32" else 1e-4
        assert errors(C, Cr)[1] <= tol and errors(n, nr)[1] <= tol
    else:
        assert errors(C, Cr)[1] <= STATE_REL_L2 and errors(n, nr)[1] <= STATE_REL_L2
    assert np.max(np.abs(m - mr)) <= STATE_M_ABS


def test_tiny_fp32_full():
    w = syn.TINY
    inp = _inputs(w)
    h, C, n, m = gpu_fwd(inp, 64, w.fgate)
    hr, Cr, nr, mr = _oracle(w, inp)
    assert_close(h, hr, "f32")
    _check_state(C, n, m, Cr, nr, mr, "f32")


@pytest.mark.parametrize("path", [xb.PATH_AUTO, xb.PATH_SIMT])
def test_small_bf16_full(path):
    w = syn.SMALL
    inp = _inputs(w)
    h, C, n, m = gpu_fwd(inp, 64, w.fgate, path)
    hr, Cr, nr, mr = _oracle(w, inp)
    assert_close(h, hr, "bf16", elementwise=fp32_arith(w.DH, 64, "bf16", path))
    _check_state(C, n, m, Cr, nr, mr, "bf16")


@pytest.mark.parametrize("chunk", [64, 128])
def test_block_bf16_full(chunk):
    w = syn.BLOCK
    inp = _inputs(w)
    h, C, n, m = gpu_fwd(inp, chunk, w.fgate)
    hr, Cr, nr, mr = _oracle(w, inp)
    assert_close(h, hr, "bf16", elementwise=fp32_arith(w.DH, chunk, "bf16"))
    _check_state(C, n, m, Cr, nr, mr, "bf16")


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_long_bf16_full_with_final_state(chunk):
    w = syn.LONG
    inp = _inputs(w)
    h, C, n, m = gpu_fwd(inp, chunk, w.fgate)
    hr, Cr, nr, mr = _oracle(w, inp)
    assert_close(h, hr, "bf16", elementwise=fp32_arith(w.DH, chunk, "bf16"))
    _check_state(C, n, m, Cr, nr, mr, "bf16")


RAGGED = [
    # (B, NH, S, DH, dtype, fgate, chunk, segments)
    (2, 3, 333, 48, "f32", "sigmoid", 40, 0),
    (2, 3, 333, 48, "f32", "sigmoid", 40, 3),
    (1, 2, 517, 128, "bf16", "sigmoid", 64, 1),
    (1, 2, 517, 128, "bf16", "sigmoid", 64, 4),
    (1, 2, 517, 128, "bf16", "exp", 128, 3),
    (3, 1, 700, 64, "bf16", "sigmoid", 256, 2),
    (1, 1, 300, 512, "bf16", "exp", 64, 2),
    (1, 3, 129, 16, "f32", "exp", 1, 5),
    (2, 2, 95, 256, "bf16", "sigmoid", 64, 0),
    (1, 1, 1, 64, "bf16", "sigmoid", 64, 0),
    (1, 1, 1, 32, "f32", "sigmoid", 1024, 0),
]


@pytest.mark.parametrize("case", RAGGED, ids=lambda c: "x".join(map(str, c)))
def test_ragged_multitile_segments(case):
    B, NH, S, DH, dtype, fgate, chunk, seg = case
    base = syn.BLOCK if fgate == "exp" else syn.SMALL
    w = syn.custom("ragged", B, NH, S, DH, base, dtype=dtype, seed=S + DH)
    inp = syn.fwd_inputs(w)
    hr, Cr, nr, mr = oracle_fwd(inp, fgate)
    tol = "f32_wide" if (dtype == "f32" and fgate == "exp") else dtype
    for path in (xb.PATH_AUTO, xb.PATH_SIMT):
        h, C, n, m = gpu_fwd(inp, chunk, fgate, path, seg)
        assert_close(h, hr, tol, elementwise=tol != "bf16" or fp32_arith(DH, chunk, dtype, path))
        _check_state(C, n, m, Cr, nr, mr, tol)


@pytest.mark.parametrize("dtype,chunk", [("f32", 32), ("bf16", 64)])
def test_initial_state(dtype, chunk):
    w = syn.custom("init", 2, 2, 200, 64, syn.SMALL, dtype=dtype, seed=3)
    inp = syn.fwd_inputs(w)
    g = torch.Generator().manual_seed(17)
    C0 = torch.randn(2, 2, 64, 64, generator=g) * 0.1
    n0 = torch.randn(2, 2, 64, generator=g) * 0.1
    m0 = torch.randn(2, 2, generator=g)
    hr, Cr, nr, mr = oracle_fwd(inp, "sigmoid", C0, n0, m0)
    for seg in (0, 3):
        h, C, n, m = gpu_fwd(inp, chunk, "sigmoid", xb.PATH_AUTO, seg, C0, n0, m0)
        assert_close(h, hr, dtype, elementwise=dtype != "bf16" or fp32_arith(64, chunk, dtype))
        _check_state(C, n, m, Cr, nr, mr, dtype)


def test_empty_sequence_passes_state_through():
    w = syn.custom("empty", 2, 3, 0, 32, syn.SMALL, dtype="f32")
    inp = syn.fwd_inputs(w)
    g = torch.Generator().manual_seed(1)
    C0, n0, m0 = torch.randn(2, 3, 32, 32, generator=g), torch.randn(2, 3, 32, generator=g), \
        torch.randn(2, 3, generator=g)
    h, C, n, m = gpu_fwd(inp, 64, "sigmoid", C0=C0, n0=n0, m0=m0)
    assert h.shape == (2, 3, 0, 32)
    assert np.array_equal(C, C0.numpy()) and np.array_equal(n, n0.numpy()) and np.array_equal(m, m0.numpy())
    h, C, n, m = gpu_fwd(inp, 64, "sigmoid")
    assert not C.any() and not n.any() and not m.any()
