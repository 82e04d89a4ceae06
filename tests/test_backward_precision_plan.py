"""Precision plan for a tensor-core backward, checked on the float64 chunkwise
model (``tests/backward_chunkwise_model.py``) against the gradient oracle.

Rounding the operands of each product of the backward to a tensor-core type
(round to nearest) and keeping fp32-or-better accumulation, the plan is:
  * dP = dnum' v^T and the reverse-state update (dnum' g)^T q: bf16 operands;
  * W o dP and W o S (the masked intra weights times dP or the scores) as the
    sum of a bf16 high part and a bf16 low part -- with them in plain bf16 the
    ftilde gradient reaches ~9e-3 of its scale, with the split ~5e-6;
  * products with the fp32 states (C'_prev^T dnum', dC~ khat, dC~^T v): tf32.
The gradients then stay within 5e-3 of max(1, max |ref|) and 5e-3 relative L2,
inside the bf16 path's tolerances, on ordinary and on wide input gates."""
import numpy as np
import pytest
import torch

import oracle.backward as bw
from backward_chunkwise_model import backward as chunkwise_backward


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float64)).to(torch.bfloat16).double().numpy()


def _tf32(x):
    a = np.ascontiguousarray(x, np.float32).copy()
    u = a.view(np.uint32)
    u += 0x0FFF + ((u >> 13) & 1)          # round to nearest even at 10 mantissa bits
    u &= 0xFFFFE000
    return a.astype(np.float64)


def _bf16_mm(a, b):
    return _bf16(a) @ _bf16(b)


def _split_mm(a, b):
    hi = _bf16(a)
    return hi @ _bf16(b) + _bf16(a - hi) @ _bf16(b)


def _tf32_mm(a, b):
    return _tf32(a) @ _tf32(b)


PLAN = {"dP": _bf16_mm, "dCb_update": _bf16_mm, "G_khat": _split_mm, "G_q": _split_mm,
        "WS_dnum": _split_mm, "Cprev": _tf32_mm, "dCb_terms": _tf32_mm}


def test_tf32_rounding_helper():
    x = np.array([1.0, 1.0 + 2.0 ** -10, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11])
    np.testing.assert_array_equal(_tf32(x), [1.0, 1.0 + 2.0 ** -10, 1.0, 1.0 + 2.0 ** -9])


@pytest.mark.parametrize("fgate,wide", [("sigmoid", False), ("exp", True)])
def test_tensor_core_precision_plan_keeps_gradients_within_budget(fgate, wide):
    g = np.random.default_rng(0)
    shp = (1, 2, 192, 64)
    d = dict(q=_bf16(g.normal(0, 1, shp)), k=_bf16(g.normal(0, 1, shp)),
             v=_bf16(g.normal(0, 1, shp)), i_pre=g.normal(0, 3 if wide else 1, shp[:3]),
             f_pre=(g.normal(3, 1, shp[:3]) if fgate == "sigmoid"
                    else g.normal(-0.05, 0.1, shp[:3])),
             o_pre=g.normal(0, 1, shp))
    dh = _bf16(g.normal(0, 1, shp))
    ref = bw.grads(*(d[nm] for nm in bw.GRAD_NAMES), dh, fgate)[1]
    got = chunkwise_backward(*(d[nm] for nm in bw.GRAD_NAMES), dh, 64, fgate, ops=PLAN)
    for nm in bw.GRAD_NAMES:
        r = ref[nm]
        err = float(np.max(np.abs(got[nm] - r))) / max(1.0, float(np.max(np.abs(r))))
        rel = float(np.linalg.norm(got[nm] - r) / np.linalg.norm(r))
        assert err <= 5e-3 and rel <= 5e-3, f"d{nm}: {err:.2e} / {rel:.2e}"
    # the split is what keeps the forget-gate gradient accurate
    plain = dict(PLAN, G_khat=_bf16_mm, G_q=_bf16_mm)
    worse = chunkwise_backward(*(d[nm] for nm in bw.GRAD_NAMES), dh, 64, fgate, ops=plain)
    e_plain = float(np.max(np.abs(worse["f_pre"] - ref["f_pre"]))) / max(1.0, float(np.max(np.abs(ref["f_pre"]))))
    e_plan = float(np.max(np.abs(got["f_pre"] - ref["f_pre"]))) / max(1.0, float(np.max(np.abs(ref["f_pre"]))))
    assert e_plan < e_plain
