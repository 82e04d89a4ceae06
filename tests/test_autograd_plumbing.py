"""Host logic of the differentiable op (``linear_rnn_mlstm_b200.autograd``) on
the CPU: the library's forward and backward calls are replaced by stand-ins
that compute with the float64 oracles, so what is checked is the op's own
plumbing -- which tensors reach which call, in which order and dtype, the
cotangents of the final state, the chunk handed to the backward, and the
gradients that come back out of torch.autograd.  (The kernels themselves are
checked by the parity tests.)"""
import numpy as np
import pytest
import torch

import oracle
import oracle.backward as bw
from linear_rnn_mlstm_b200 import autograd as xa
from linear_rnn_mlstm_b200 import binding as xb


@pytest.fixture
def stand_ins(monkeypatch):
    calls = {}

    def fake_fwd(q, k, v, i_pre, f_pre, o_pre, chunk=64, fgate="sigmoid", **kw):
        calls["fwd"] = dict(chunk=chunk, fgate=fgate)
        h, C, n, m = oracle.fwd(q, k, v, i_pre, f_pre, o_pre, fgate)
        return (torch.from_numpy(h).to(q.dtype), torch.from_numpy(C).float(),
                torch.from_numpy(n).float(), torch.from_numpy(m).float())

    def fake_bwd(q, k, v, i_pre, f_pre, o_pre, dh, dC=None, dn=None, chunk=64, fgate="sigmoid"):
        calls["bwd"] = dict(chunk=chunk, fgate=fgate, dh_dtype=dh.dtype,
                            dC=None if dC is None else dC.clone(),
                            dn=None if dn is None else dn.clone())
        _, g = bw.grads(q, k, v, i_pre, f_pre, o_pre, dh, fgate,
                        dC=None if dC is None else dC.numpy(), dn=None if dn is None else dn.numpy())
        out = {"dq": g["q"], "dk": g["k"], "dv": g["v"], "di": g["i_pre"], "df": g["f_pre"],
               "do": g["o_pre"]}
        dt = {"dq": q.dtype, "dk": k.dtype, "dv": v.dtype}
        return {nm: torch.from_numpy(x).to(dt.get(nm, torch.float32)) for nm, x in out.items()}

    monkeypatch.setattr(xb, "mlstm_fwd", fake_fwd)
    monkeypatch.setattr(xb, "mlstm_bwd", fake_bwd)
    return calls


def _inputs(seed=0, B=1, NH=2, S=9, DH=8, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    shp = (B, NH, S, DH)
    mk = lambda *s, mu=0.0: (torch.randn(*s, generator=g) + mu)
    x = dict(q=mk(*shp).to(dtype), k=mk(*shp).to(dtype), v=mk(*shp).to(dtype),
             i_pre=mk(*shp[:3]), f_pre=mk(*shp[:3], mu=3.0), o_pre=mk(*shp))
    return {nm: t.detach().requires_grad_(True) for nm, t in x.items()}


NAMES = ("q", "k", "v", "i_pre", "f_pre", "o_pre")


def test_gradients_of_h_and_final_state_reach_every_input(stand_ins):
    x = _inputs()
    h, C, n, m = xa.mlstm_cell(*(x[nm] for nm in NAMES), chunk=128, fgate="sigmoid")
    g = torch.Generator().manual_seed(7)
    wh, wC, wn = (torch.randn(t.shape, generator=g) for t in (h, C, n))
    ((h * wh).sum() + (C * wC).sum() + (n * wn).sum()).backward()
    _, ref = bw.grads(*(x[nm].detach() for nm in NAMES), wh.numpy(), "sigmoid",
                      dC=wC.numpy(), dn=wn.numpy())
    for nm in NAMES:
        np.testing.assert_allclose(x[nm].grad.numpy(), ref[nm], rtol=1e-5, atol=1e-6, err_msg=nm)
    assert stand_ins["fwd"]["chunk"] == 128
    assert stand_ins["bwd"]["chunk"] == xa.BWD_MAX_CHUNK       # the backward's chunk limit
    assert not m.requires_grad


def test_unused_final_state_gets_zero_cotangents(stand_ins):
    x = _inputs(seed=1)
    h, C, n, m = xa.mlstm_cell(*(x[nm] for nm in NAMES), chunk=16, fgate="exp")
    h.sum().backward()
    got = stand_ins["bwd"]
    assert got["chunk"] == 16 and got["fgate"] == "exp"
    assert got["dC"] is not None and not torch.any(got["dC"])
    _, ref = bw.grads(*(x[nm].detach() for nm in NAMES), np.ones(h.shape), "exp")
    for nm in NAMES:
        np.testing.assert_allclose(x[nm].grad.numpy(), ref[nm], rtol=1e-5, atol=1e-6, err_msg=nm)


def test_bf16_inputs_get_bf16_gradients(stand_ins):
    x = _inputs(seed=2, dtype=torch.bfloat16)
    h, C, n, m = xa.mlstm_cell(*(x[nm] for nm in NAMES))
    assert h.dtype == torch.bfloat16
    h.float().sum().backward()
    assert stand_ins["bwd"]["dh_dtype"] == torch.bfloat16
    for nm in ("q", "k", "v"):
        assert x[nm].grad.dtype == torch.bfloat16
    for nm in ("i_pre", "f_pre", "o_pre"):
        assert x[nm].grad.dtype == torch.float32
