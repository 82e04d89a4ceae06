"""The seeded input recipe (``linear_rnn_mlstm_b200.synthetic``) matches the
workloads it stands for: shapes and dtypes of the five configurations, the
gate distributions (sample moments within a few standard errors), q/k/v
rounded to bf16 on the host for bf16 workloads, and determinism of the draws
(the same seed gives the same tensors; a decode step can be drawn alone)."""
import math

import pytest
import torch

from linear_rnn_mlstm_b200 import synthetic as syn

SHAPES = {"tiny": (1, 2, 64, 16, "f32", "sigmoid"), "small": (4, 4, 1024, 64, "bf16", "sigmoid"),
          "block": (4, 4, 2048, 512, "bf16", "exp"), "long": (1, 8, 16384, 256, "bf16", "sigmoid")}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_workload_shapes_and_gate_kinds(name):
    w = syn.WORKLOADS[name]
    B, NH, S, DH, dt, fg = SHAPES[name]
    assert (w.B, w.NH, w.S, w.DH, w.dtype, w.fgate) == (B, NH, S, DH, dt, fg)


def _moments_ok(x, mu, sd, tol_se=6.0):
    x = x.double().flatten()
    n = x.numel()
    m, s = float(x.mean()), float(x.std())
    return abs(m - mu) <= tol_se * sd / math.sqrt(n) and abs(s - sd) <= tol_se * sd / math.sqrt(2 * n)


@pytest.mark.parametrize("name", ["tiny", "small", "block", "long"])
def test_inputs_follow_the_stated_distributions(name):
    w = syn.WORKLOADS[name]
    x = syn.fwd_inputs(w, S=min(w.S, 256))
    B, NH, S, DH = w.B, w.NH, min(w.S, 256), w.DH
    qdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    for nm in ("q", "k", "v"):
        assert x[nm].shape == (B, NH, S, DH) and x[nm].dtype == qdt
    assert x["o_pre"].shape == (B, NH, S, DH) and x["o_pre"].dtype == torch.float32
    assert x["i_pre"].shape == (B, NH, S) and x["f_pre"].shape == (B, NH, S)
    assert _moments_ok(x["i_pre"], w.i_mu, w.i_sd)
    assert _moments_ok(x["f_pre"], w.f_mu, w.f_sd)
    assert _moments_ok(x["o_pre"], 0.0, 1.0)
    for nm in ("q", "k", "v"):                   # N(0,1) (bf16 rounding moves them < 1 %)
        assert _moments_ok(x[nm], 0.0, 1.0, tol_se=6.0 + 0.01 * math.sqrt(x[nm].numel()))


def test_the_named_distributions_of_the_pages_workloads():
    assert (syn.SMALL.f_mu, syn.SMALL.f_sd, syn.SMALL.i_sd) == (3.0, 1.0, 1.0)
    assert (syn.BLOCK.f_mu, syn.BLOCK.f_sd, syn.BLOCK.i_sd) == (-0.05, 0.1, 3.0)
    assert (syn.LONG.f_mu, syn.LONG.f_sd, syn.LONG.i_sd) == (4.0, 1.0, 1.0)
    d = syn.DECODE
    assert (d.B, d.NH, d.DH, d.steps, d.prefill_S, d.prefill_chunk) == (256, 8, 512, 1024, 512, 64)


def test_draws_are_deterministic_and_seeded():
    w = syn.custom("c", 1, 2, 40, 16, syn.SMALL)
    a, b, c = syn.fwd_inputs(w, seed=5), syn.fwd_inputs(w, seed=5), syn.fwd_inputs(w, seed=6)
    for nm in a:
        assert torch.equal(a[nm], b[nm])
    assert not torch.equal(a["q"], c["q"])
    d = syn.DecodeWorkload("d", 2, 2, 16, 5, 0)
    s3a, s3b = syn.step_inputs(d, 3), syn.step_inputs(d, 3)
    for nm in s3a:
        assert torch.equal(s3a[nm], s3b[nm])
    assert not torch.equal(syn.step_inputs(d, 2)["q"], s3a["q"])


def test_bf16_rounding_happens_on_the_host():
    w = syn.custom("c", 1, 1, 8, 16, syn.SMALL)
    q = syn.fwd_inputs(w)["q"]
    assert q.dtype == torch.bfloat16 and q.device.type == "cpu"
