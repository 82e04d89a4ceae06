"""GPU parity of the sLSTM forward (``xlstm_slstm_fwd``) against the float64
sLSTM oracle (``oracle.slstm``), with the tolerance of the host-emulation test
(``test_slstm_emulation.py``, which checks the same per-unit code on the CPU):
max |got - ref| / max(1, max |ref|) <= 1e-5 on h and the final (c', n', h),
1e-5 absolute on m.  Named to be collected after the mLSTM parity tests."""
import pytest
import torch

from linear_rnn_mlstm_b200 import binding as xb

from test_slstm_emulation import compare, inputs, oracle_run

pytestmark = pytest.mark.gpu

# DH 64, 128, 256 and 512 run on the cluster kernel (DH / 32 CTAs per head, the
# recurrent blocks in registers, at DH 512 half of them in shared memory; 16-step
# input stages: S below one stage, across several and with a ragged last one);
# the other head sizes on the per-unit kernel.
CASES = [(1, 2, 17, 16, "sigmoid", False), (2, 3, 9, 8, "exp", False),
         (1, 2, 33, 48, "sigmoid", True), (2, 4, 256, 64, "sigmoid", False),
         (1, 2, 40, 512, "exp", True), (1, 1, 1, 4, "exp", True),
         (1, 2, 100, 128, "exp", True), (2, 2, 70, 256, "sigmoid", True),
         (1, 1, 5, 256, "exp", False), (3, 1, 33, 64, "exp", True), (2, 1, 37, 512, "sigmoid", False)]


@pytest.mark.parametrize("B,NH,S,DH,fgate,state", CASES,
                         ids=[f"B{c[0]}NH{c[1]}S{c[2]}DH{c[3]}-{c[4]}{'-state' if c[5] else ''}"
                              for c in CASES])
def test_slstm_matches_oracle(cuda_lib, B, NH, S, DH, fgate, state):
    x = inputs(B, NH, S, DH, fgate, seed=S + DH, state=state)
    d = {k: torch.from_numpy(v).cuda().contiguous() for k, v in x.items()}
    got = xb.slstm_fwd(d["zx"], d["ix"], d["fx"], d["ox"], d["R"], fgate,
                       d.get("c0"), d.get("n0"), d.get("m0"), d.get("h0"))
    torch.cuda.synchronize()
    assert xb.xlstm_device_status(torch.cuda.current_stream().cuda_stream) == xb.OK
    compare([t.cpu().numpy() for t in got], oracle_run(x, fgate))
