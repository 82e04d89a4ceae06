"""Failure detection without a GPU fault: every device-side wait in the kernels
is bounded; when it runs out the kernel latches the device status word and
returns, and the host reads the word.  The self-test entry point waits on a
barrier nothing completes, so the path runs for real while the context stays
usable."""
import pytest
import torch

from linear_rnn_mlstm_b200 import binding as xb
from linear_rnn_mlstm_b200 import synthetic as syn

from parity import assert_close, gpu_fwd, oracle_fwd


def test_selftest_rejects_out_of_range_limits_before_device_work():
    assert xb.xlstm_selftest_wait_timeout(0, None) == xb.ERR_SHAPE
    assert xb.xlstm_selftest_wait_timeout(1000001, None) == xb.ERR_SHAPE


@pytest.mark.gpu
def test_bounded_wait_runs_out_latches_status_and_the_context_survives():
    stream = torch.cuda.current_stream().cuda_stream
    assert xb.xlstm_device_status(stream) == xb.OK          # start clean
    assert xb.xlstm_selftest_wait_timeout(2000, stream) == xb.OK
    assert xb.xlstm_device_status(stream) == xb.ERR_TIMEOUT
    assert xb.xlstm_device_status(stream) == xb.OK          # reading clears the word
    # the context is still usable: a forward on both paths passes parity afterwards
    w = syn.custom("after", 1, 2, 130, 128, syn.SMALL, seed=9)
    inp = syn.fwd_inputs(w)
    hr = oracle_fwd(inp, "sigmoid")[0]
    for path in (xb.PATH_TENSOR, xb.PATH_SIMT):
        h = gpu_fwd(inp, 64, "sigmoid", path)[0]
        assert_close(h, hr, "bf16")
