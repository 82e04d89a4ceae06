"""The binding's torch conveniences check their tensors before any library
call, on the CPU: tensors off the GPU, wrong shapes and wrong dtypes raise a
Python error (no fallback computes anything on the host)."""
import pytest
import torch

from linear_rnn_mlstm_b200 import binding as xb


def _fwd_args(B=1, NH=2, S=8, DH=16, dtype=torch.float32):
    shp = (B, NH, S, DH)
    return [torch.zeros(shp, dtype=dtype) for _ in range(3)] + \
        [torch.zeros(shp[:3]), torch.zeros(shp[:3]), torch.zeros(shp)]


def test_forward_refuses_host_tensors():
    with pytest.raises(ValueError, match="CUDA tensor"):
        xb.mlstm_fwd(*_fwd_args())


def test_step_refuses_host_tensors():
    q = torch.zeros(1, 2, 16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        xb.mlstm_step(q, q, q, torch.zeros(1, 2), torch.zeros(1, 2), q,
                      torch.zeros(1, 2, 16, 16), torch.zeros(1, 2, 16), torch.zeros(1, 2))


def test_backward_refuses_host_tensors():
    a = _fwd_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        xb.mlstm_bwd(*a, torch.zeros_like(a[0]))


def test_epilogue_refuses_host_tensors():
    h = torch.zeros(1, 2, 8, 16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        xb.mlstm_headnorm_gate(h, torch.ones(32), torch.zeros(32), torch.zeros(1, 8, 32))


def test_slstm_refuses_host_tensors():
    x = torch.zeros(1, 2, 4, 16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        xb.slstm_fwd(x, x, x, x, torch.zeros(2, 4, 16, 16))


def test_unsupported_dtype_is_a_type_error():
    a = _fwd_args(dtype=torch.float16)
    with pytest.raises(TypeError):
        xb.mlstm_fwd(*a)
