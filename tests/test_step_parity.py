"""GPU decode step vs the float64 oracle.

(1) The step alone: the same fp32 state is handed to both sides.
(2) Prefill then steps, end to end, bf16.
(3) The full decode workload (B=256, NH=8, DH=512, prefill S=512, 1024 steps)
    in the launch configuration the benchmark times, checked on a seeded
    sample of 32 heads (heads are independent: section 2.3 of the paper).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_mlstm_b200 import binding as xb
from linear_rnn_mlstm_b200 import synthetic as syn

from parity import STATE_M_ABS, TOL, assert_close, errors, fp32_arith, to_cuda

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("DH,fgate", [(64, "sigmoid"), (48, "exp"), (512, "sigmoid"), (16, "sigmoid"),
                                      (128, "exp"), (256, "sigmoid")])
def test_step_alone_fp32(DH, fgate):
    d = syn.DecodeWorkload("d", 2, 3, DH, 8, 0, dtype="f32", fgate=fgate, seed=DH)
    g = torch.Generator().manual_seed(DH)
    C = torch.randn(2, 3, DH, DH, generator=g) * 0.2
    n = torch.randn(2, 3, DH, generator=g) * 0.2
    m = torch.randn(2, 3, generator=g)
    Cg, ng, mg = C.cuda(), n.cuda(), m.cuda()
    Cr, nr, mr = C.double().numpy(), n.double().numpy(), m.double().numpy()
    for t in range(d.steps):
        inp = syn.step_inputs(d, t)
        x = to_cuda(inp)
        h = xb.mlstm_step(x["q"], x["k"], x["v"], x["i_pre"], x["f_pre"], x["o_pre"], Cg, ng, mg,
                          fgate=fgate)
        hr, Cr, nr, mr = oracle.step(inp["q"], inp["k"], inp["v"], inp["i_pre"], inp["f_pre"],
                                     inp["o_pre"], Cr, nr, mr, fgate)
        torch.cuda.synchronize()
        # the exponential forget gate is the wide-gate regime of the fp32 tolerance
        # (a plain fp32 evaluation of these steps already reaches ~1.4e-5 per element)
        assert_close(h.cpu().numpy(), hr, "f32_wide" if fgate == "exp" else "f32")
    tol = 1e-4 if fgate == "exp" else 1e-5
    assert errors(Cg.cpu().numpy(), Cr)[1] <= tol
    assert errors(ng.cpu().numpy(), nr)[1] <= tol
    assert np.max(np.abs(mg.cpu().numpy() - mr)) <= 1e-5
    assert xb.xlstm_device_status(_stream()) == xb.OK


def test_prefill_then_steps_bf16():
    d = syn.DecodeWorkload("d", 2, 2, 256, 24, 200, prefill_chunk=64, seed=5)
    pre = syn.fwd_inputs(d.prefill())
    x = to_cuda(pre)
    _, Cg, ng, mg = xb.mlstm_fwd(x["q"], x["k"], x["v"], x["i_pre"], x["f_pre"], x["o_pre"],
                                 chunk=64, fgate=d.fgate)
    _, Cr, nr, mr = oracle.fwd(pre["q"], pre["k"], pre["v"], pre["i_pre"], pre["f_pre"],
                               pre["o_pre"], d.fgate)
    hs, hrs = [], []
    for t in range(d.steps):
        inp = syn.step_inputs(d, t)
        y = to_cuda(inp)
        hs.append(xb.mlstm_step(y["q"], y["k"], y["v"], y["i_pre"], y["f_pre"], y["o_pre"],
                                Cg, ng, mg, fgate=d.fgate).float().cpu().numpy())
        hr, Cr, nr, mr = oracle.step(inp["q"], inp["k"], inp["v"], inp["i_pre"], inp["f_pre"],
                                     inp["o_pre"], Cr, nr, mr, d.fgate)
        hrs.append(hr)
    torch.cuda.synchronize()
    # the steps are fp32 arithmetic; so is the prefill when it runs on the SIMT kernels
    assert_close(np.stack(hs), np.stack(hrs), "bf16", elementwise=fp32_arith(d.DH, 64, "bf16"))
    assert errors(Cg.cpu().numpy(), Cr)[1] <= 1e-2
    assert np.max(np.abs(mg.cpu().numpy() - mr)) <= STATE_M_ABS
    assert xb.xlstm_device_status(_stream()) == xb.OK


def sample_heads(B, NH, count, seed=0):
    """A seeded sample of (b, h) pairs that always includes the first and last head."""
    rng = np.random.default_rng(seed)
    flat = rng.choice(B * NH, size=count, replace=False)
    flat[0], flat[1] = 0, B * NH - 1
    flat = np.unique(flat)
    return [(int(f) // NH, int(f) % NH) for f in flat]


def test_decode_workload_full_size_sampled_heads():
    d = syn.DECODE
    heads = sample_heads(d.B, d.NH, 32)
    bi = torch.tensor([b for b, _ in heads])
    hi = torch.tensor([h for _, h in heads])
    pick = lambda t: t[bi, hi]
    pre = syn.fwd_inputs(d.prefill())
    x = to_cuda(pre)
    _, Cg, ng, mg = xb.mlstm_fwd(x["q"], x["k"], x["v"], x["i_pre"], x["f_pre"], x["o_pre"],
                                 chunk=d.prefill_chunk, fgate=d.fgate)
    del x
    sub = {k: pick(v).unsqueeze(0) for k, v in pre.items()}       # [1, nsample, ...]
    _, Cr, nr, mr = oracle.fwd(sub["q"], sub["k"], sub["v"], sub["i_pre"], sub["f_pre"],
                               sub["o_pre"], d.fgate)
    hs, hrs = [], []
    for t in range(d.steps):
        inp = syn.step_inputs(d, t)
        y = to_cuda(inp)
        h = xb.mlstm_step(y["q"], y["k"], y["v"], y["i_pre"], y["f_pre"], y["o_pre"],
                          Cg, ng, mg, fgate=d.fgate)
        hs.append(pick(h).float().cpu().numpy())
        s = {k: pick(v).unsqueeze(0) for k, v in inp.items()}
        hr, Cr, nr, mr = oracle.step(s["q"], s["k"], s["v"], s["i_pre"], s["f_pre"], s["o_pre"],
                                     Cr, nr, mr, d.fgate)
        hrs.append(hr[0])
    torch.cuda.synchronize()
    assert_close(np.stack(hs), np.stack(hrs), "bf16",
                 elementwise=fp32_arith(d.DH, d.prefill_chunk, "bf16"))
    assert errors(pick(Cg).cpu().numpy(), Cr[0])[1] <= 1e-2
    assert np.max(np.abs(pick(mg).cpu().numpy() - mr[0])) <= STATE_M_ABS
    assert xb.xlstm_device_status(_stream()) == xb.OK
