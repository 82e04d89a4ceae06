"""The forward entry point that allocates nothing (xlstm_mlstm_fwd_noalloc).

Some callers cannot allocate device memory: code that reaches the library only
through its C ABI with no device allocator of its own, or a serving loop that
must not call cudaMalloc (which can synchronise the device, fail under memory
pressure, or stall).  For them the library keeps its forward scratch in one
built-in device array.  These tests call that entry point through the C ABI
twice in a row, on different inputs, and check each result against the
ordinary entry point (caller-provided workspace) with the tolerances the other
parity tests use.  The file is named to be collected last.
"""
import pytest
import torch

from linear_rnn_mlstm_b200 import binding as xb
from linear_rnn_mlstm_b200 import synthetic as syn

from parity import assert_close, errors

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else t.data_ptr()


def _run_both(w, chunk):
    """Returns (outputs of the ordinary entry point, outputs of the no-alloc one)."""
    x = {k: v.cuda().contiguous() for k, v in syn.fwd_inputs(w).items()}
    dt = xb.BF16 if w.dtype == "bf16" else xb.F32
    fg = xb.FGATE_EXP if w.fgate == "exp" else xb.FGATE_SIGMOID
    stream = torch.cuda.current_stream().cuda_stream
    st, need = xb.xlstm_mlstm_fwd_workspace_size(w.B, w.NH, w.S, w.DH, chunk, dt)
    assert st == xb.OK and 0 < need <= xb.NOALLOC_SCRATCH_BYTES
    outs = []
    for use_noalloc in (False, True):
        h = torch.empty_like(x["q"])
        C = torch.empty((w.B, w.NH, w.DH, w.DH), dtype=torch.float32, device="cuda")
        n = torch.empty((w.B, w.NH, w.DH), dtype=torch.float32, device="cuda")
        m = torch.empty((w.B, w.NH), dtype=torch.float32, device="cuda")
        args = [_ptr(x[k]) for k in ("q", "k", "v", "i_pre", "f_pre", "o_pre")] + \
            [h.data_ptr(), None, None, None, C.data_ptr(), n.data_ptr(), m.data_ptr(),
             w.B, w.NH, w.S, w.DH, chunk, dt, fg]
        if use_noalloc:
            st = xb.xlstm_mlstm_fwd_noalloc(*args, stream)
        else:
            ws = torch.empty(need, dtype=torch.uint8, device="cuda")
            st = xb.xlstm_mlstm_fwd(*args, ws.data_ptr(), need, stream)
        assert st == xb.OK, xb.status_string(st)
        torch.cuda.synchronize()
        outs.append([t.float().cpu().numpy() for t in (h, C, n, m)])
    assert xb.xlstm_device_status(stream) == xb.OK
    return outs


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    # two different problems back to back: the second call reuses the built-in
    # scratch that the first one left behind
    cases = [(syn.custom("noalloc-a", 1, 4, 2048, 128, syn.SMALL, seed=11), 64, "bf16"),
             (syn.custom("noalloc-b", 2, 3, 777, 64, syn.SMALL, dtype="f32", seed=12), 40, "f32")]
    for w, chunk, tol in cases:
        ref, got = _run_both(w, chunk)
        assert_close(got[0], ref[0], tol, "h")
        for a, b in zip(got[1:], ref[1:]):
            assert errors(a, b)[1] <= (1e-5 if tol == "f32" else 1e-2)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # needs more than the built-in scratch (per-token prefix sums alone exceed it):
    # rejected on the host, before any device work, so fake addresses are never used
    fake = 1 << 40
    st, need = xb.xlstm_mlstm_fwd_workspace_size(1, 256, 65536, 64, 64, xb.BF16)
    assert st == xb.OK and need > xb.NOALLOC_SCRATCH_BYTES
    st = xb.xlstm_mlstm_fwd_noalloc(fake, fake, fake, fake, fake, fake, fake, None, None, None,
                                    None, None, None, 1, 256, 65536, 64, 64, xb.BF16,
                                    xb.FGATE_SIGMOID, None)
    assert st == xb.ERR_WORKSPACE
