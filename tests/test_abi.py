"""Host-side checks of the C ABI: the library loads, exports every entry point
the header declares, and rejects bad arguments before touching any device.
No test here launches GPU work (fake device addresses are only ever passed
where validation must reject them first)."""
import ctypes
import os
import re

import pytest

from linear_rnn_mlstm_b200 import binding as xb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "xlstm_mlstm.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(xlstm_\w+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    assert set(_declared()) == set(xb.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(xb.LIB_PATH)
    missing = [name for name in _declared() if not hasattr(lib, name)]
    assert not missing, missing


def test_abi_version_and_status_strings():
    assert xb.xlstm_abi_version() == 1
    for s in range(10):
        assert xb.status_string(s) and "unknown" not in xb.status_string(s)
    assert "unknown" in xb.status_string(99)


@pytest.mark.parametrize("args,expect", [
    ((1, 1, 64, 64, 64, xb.BF16), xb.OK),
    ((1, 1, 64, 64, 32, xb.BF16), xb.ERR_CHUNK),      # bf16 chunk must be 64/128/256
    ((1, 1, 64, 64, 0, xb.F32), xb.ERR_CHUNK),
    ((1, 1, 64, 64, 2048, xb.F32), xb.ERR_CHUNK),
    ((1, 1, 64, 24, 64, xb.F32), xb.ERR_SHAPE),       # DH not a multiple of 16
    ((1, 1, 64, 528, 64, xb.F32), xb.ERR_SHAPE),      # DH > 512
    ((-1, 1, 64, 64, 64, xb.F32), xb.ERR_SHAPE),
    ((1, 1, -5, 64, 64, xb.F32), xb.ERR_SHAPE),
    ((300, 300, 64, 64, 64, xb.F32), xb.ERR_SHAPE),   # B * NH beyond one grid dimension
    ((1, 1, 64, 64, 64, 7), xb.ERR_DTYPE),
])
def test_workspace_size_validation(args, expect):
    st, _ = xb.xlstm_mlstm_fwd_workspace_size(*args)
    assert st == expect


def test_workspace_size_grows_with_segments_and_is_zero_for_empty():
    st, n1 = xb.xlstm_mlstm_fwd_workspace_size(1, 2, 1024, 64, 64, xb.F32, xb.PATH_SIMT, 1)
    st2, n4 = xb.xlstm_mlstm_fwd_workspace_size(1, 2, 1024, 64, 64, xb.F32, xb.PATH_SIMT, 4)
    assert st == st2 == xb.OK and n4 > n1 > 0
    # three extra segment summaries of DH*DH + DH floats per head, plus segment stats
    assert n4 - n1 >= 3 * 2 * (64 * 64 + 64) * 4
    st, n0 = xb.xlstm_mlstm_fwd_workspace_size(1, 2, 0, 64, 64, xb.F32)
    assert st == xb.OK and n0 == 0


FAKE = 1 << 40          # an aligned address; validation must reject before use


def _fwd(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, i_pre=FAKE, f_pre=FAKE, o_pre=FAKE, h=FAKE, C0=None,
             n0=None, m0=None, C_out=None, n_out=None, m_out=None, B=1, NH=1, S=64, DH=64,
             chunk=64, dt=xb.F32, fg=xb.FGATE_SIGMOID, workspace=FAKE, workspace_bytes=0,
             stream=None)
    a.update(over)
    return xb.xlstm_mlstm_fwd(**a)


@pytest.mark.parametrize("over,expect", [
    (dict(q=None), xb.ERR_NULL),
    (dict(o_pre=None), xb.ERR_NULL),
    (dict(h=None), xb.ERR_NULL),
    (dict(k=FAKE + 8), xb.ERR_ALIGN),
    (dict(C0=FAKE + 4), xb.ERR_ALIGN),
    (dict(fg=5), xb.ERR_DTYPE),
    (dict(dt=xb.BF16, chunk=100), xb.ERR_CHUNK),
    (dict(DH=40), xb.ERR_SHAPE),
    (dict(workspace_bytes=16), xb.ERR_WORKSPACE),       # far smaller than required
    (dict(workspace=None, workspace_bytes=1 << 30), xb.ERR_WORKSPACE),
    (dict(segments=-1), xb.ERR_UNSUPPORTED),
    (dict(path=7), xb.ERR_UNSUPPORTED),
    (dict(path=xb.PATH_TENSOR, dt=xb.F32), xb.ERR_UNSUPPORTED),
    (dict(B=0), xb.OK),                                  # no heads: a no-op
    (dict(NH=0, q=None), xb.OK),
])
def test_fwd_rejects_bad_arguments_before_device_work(over, expect):
    assert _fwd(**over) == expect


def _step(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, i_pre=FAKE, f_pre=FAKE, o_pre=FAKE, h=FAKE, C=FAKE, n=FAKE,
             m=FAKE, B=1, NH=1, DH=64, dt=xb.BF16, fg=xb.FGATE_SIGMOID, stream=None)
    a.update(over)
    return xb.xlstm_mlstm_step(**a)


@pytest.mark.parametrize("over,expect", [
    (dict(C=None), xb.ERR_NULL),
    (dict(m=None), xb.ERR_NULL),
    (dict(v=FAKE + 2), xb.ERR_ALIGN),
    (dict(dt=3), xb.ERR_DTYPE),
    (dict(fg=-1), xb.ERR_DTYPE),
    (dict(DH=8), xb.ERR_SHAPE),
    (dict(DH=1024), xb.ERR_SHAPE),
    (dict(B=-2), xb.ERR_SHAPE),
    (dict(B=0), xb.OK),
])
def test_step_rejects_bad_arguments_before_device_work(over, expect):
    assert _step(**over) == expect


def _headnorm(**over):
    # distinct aligned fake addresses, so that only the aliasing cases alias
    a = dict(h=FAKE, gamma=FAKE + 16, beta=FAKE + 32, skip_w=FAKE + 48, x_skip=FAKE + 64,
             z=FAKE + 80, y=FAKE + 96, B=1, NH=2, S=8, DH=64, eps=1e-5, dt=xb.BF16,
             og=xb.OGATE_SILU, stream=None)
    a.update(over)
    return xb.xlstm_mlstm_headnorm_gate(**a)


@pytest.mark.parametrize("over,expect", [
    (dict(h=None), xb.ERR_NULL),
    (dict(gamma=None), xb.ERR_NULL),
    (dict(z=None), xb.ERR_NULL),
    (dict(y=None), xb.ERR_NULL),
    (dict(skip_w=None), xb.ERR_NULL),                    # skip weight without the skip input
    (dict(x_skip=None), xb.ERR_NULL),
    (dict(z=FAKE + 88), xb.ERR_ALIGN),
    (dict(beta=FAKE + 36), xb.ERR_ALIGN),
    (dict(dt=2), xb.ERR_DTYPE),
    (dict(og=2), xb.ERR_DTYPE),
    (dict(DH=40), xb.ERR_SHAPE),
    (dict(DH=528), xb.ERR_SHAPE),
    (dict(S=-1), xb.ERR_SHAPE),
    (dict(eps=0.0), xb.ERR_UNSUPPORTED),
    (dict(eps=-1e-5), xb.ERR_UNSUPPORTED),
    (dict(eps=float("nan")), xb.ERR_UNSUPPORTED),
    (dict(eps=float("inf")), xb.ERR_UNSUPPORTED),
    (dict(y=FAKE), xb.ERR_UNSUPPORTED),                  # y is h
    (dict(y=FAKE + 80), xb.ERR_UNSUPPORTED),             # y is z
    (dict(y=FAKE + 64), xb.ERR_UNSUPPORTED),             # y is x_skip
    (dict(S=0), xb.OK),                                  # no tokens: a no-op
    (dict(B=0, h=None, y=None), xb.OK),
])
def test_headnorm_gate_rejects_bad_arguments_before_device_work(over, expect):
    assert _headnorm(**over) == expect


def _bwd(**over):
    a = dict(q=FAKE, k=FAKE + 16, v=FAKE + 32, i_pre=FAKE + 48, f_pre=FAKE + 64, o_pre=FAKE + 80,
             dh=FAKE + 96, dC=None, dn=None, dq=FAKE + 112, dk=FAKE + 128, dv=FAKE + 144,
             di=FAKE + 160, df=FAKE + 176, d_o=FAKE + 192, B=1, NH=2, S=10, DH=16, chunk=4,
             dt=xb.F32, fg=xb.FGATE_SIGMOID, workspace=FAKE + 4096, workspace_bytes=1 << 30,
             stream=None)
    a.update(over)
    return xb.xlstm_mlstm_bwd(**a)


@pytest.mark.parametrize("over,expect", [
    (dict(q=None), xb.ERR_NULL),
    (dict(dh=None), xb.ERR_NULL),
    (dict(d_o=None), xb.ERR_NULL),
    (dict(dk=FAKE + 136), xb.ERR_ALIGN),
    (dict(dC=FAKE + 4), xb.ERR_ALIGN),
    (dict(dt=5), xb.ERR_DTYPE),
    (dict(fg=2), xb.ERR_DTYPE),
    (dict(DH=40), xb.ERR_SHAPE),
    (dict(S=-3), xb.ERR_SHAPE),
    (dict(B=70000, NH=70000, S=0), xb.ERR_SHAPE),        # more heads than an int indexes
    (dict(chunk=0), xb.ERR_CHUNK),
    (dict(chunk=65), xb.ERR_CHUNK),                      # per-thread arrays hold 64 tokens
    (dict(workspace_bytes=64), xb.ERR_WORKSPACE),
    (dict(workspace=None), xb.ERR_WORKSPACE),
    (dict(dq=FAKE), xb.ERR_UNSUPPORTED),                 # an output is an input
    (dict(dv=FAKE + 112), xb.ERR_UNSUPPORTED),           # two outputs share a buffer
    (dict(di=FAKE + 4096), xb.ERR_UNSUPPORTED),          # an output is the workspace
    (dict(S=0), xb.OK),                                  # empty sequence: a no-op
    (dict(B=0, q=None), xb.OK),
])
def test_bwd_rejects_bad_arguments_before_device_work(over, expect):
    assert _bwd(**over) == expect


def test_bwd_workspace_size_matches_its_layout():
    """Per head: 8 per-token arrays, 3 per-chunk arrays, NC + 1 chunk-start
    states (C', n'), num' and dnum' per token, NC reverse states (dC, dn); each
    array padded to 64 floats."""
    pad = lambda n: (n + 63) // 64 * 64
    for B, NH, S, DH, L in ((1, 2, 10, 16, 4), (2, 3, 64, 48, 64), (1, 1, 7, 512, 1)):
        BH, NC = B * NH, (S + L - 1) // L
        sizes = [BH * S] * 8 + [BH * NC] * 3 + [BH * (NC + 1) * DH * DH, BH * (NC + 1) * DH,
                                               BH * S * DH, BH * S * DH, BH * NC * DH * DH,
                                               BH * NC * DH]
        st, n = xb.xlstm_mlstm_bwd_workspace_size(B, NH, S, DH, L, xb.F32)
        assert st == xb.OK and n == 4 * sum(pad(x) for x in sizes)
    assert xb.xlstm_mlstm_bwd_workspace_size(1, 1, 0, 16, 4, xb.F32) == (xb.OK, 0)
    assert xb.xlstm_mlstm_bwd_workspace_size(1, 1, 8, 16, 65, xb.F32)[0] == xb.ERR_CHUNK


def _slstm(**over):
    a = dict(zx=FAKE, ix=FAKE + 16, fx=FAKE + 32, ox=FAKE + 48, R=FAKE + 64, h=FAKE + 80,
             c0=None, n0=None, m0=None, h0=None, c_out=FAKE + 96, n_out=None, m_out=None,
             h_out=None, B=1, NH=2, S=5, DH=16, fg=xb.FGATE_SIGMOID, stream=None)
    a.update(over)
    return xb.xlstm_slstm_fwd(**a)


@pytest.mark.parametrize("over,expect", [
    (dict(zx=None), xb.ERR_NULL),
    (dict(R=None), xb.ERR_NULL),
    (dict(h=None), xb.ERR_NULL),
    (dict(ox=FAKE + 52), xb.ERR_ALIGN),
    (dict(h0=FAKE + 8), xb.ERR_ALIGN),
    (dict(fg=3), xb.ERR_DTYPE),
    (dict(DH=0), xb.ERR_SHAPE),
    (dict(DH=513), xb.ERR_SHAPE),
    (dict(S=-1), xb.ERR_SHAPE),
    (dict(h=FAKE), xb.ERR_UNSUPPORTED),                  # output is an input
    (dict(n_out=FAKE + 96), xb.ERR_UNSUPPORTED),         # two outputs share a buffer
    (dict(B=0, zx=None), xb.OK),
    (dict(S=0, zx=None, h=None, c_out=None), xb.OK),     # nothing to do
])
def test_slstm_rejects_bad_arguments_before_device_work(over, expect):
    assert _slstm(**over) == expect


def _seg_state(**over):
    a = dict(k=FAKE, v=FAKE, i_pre=FAKE, f_pre=FAKE, packed=FAKE, B=1, NH=2, S=200, DH=64, chunk=64,
             dt=xb.BF16, fg=xb.FGATE_SIGMOID, workspace=FAKE, workspace_bytes=0, stream=None)
    a.update(over)
    return xb.xlstm_mlstm_seg_state(**a)


@pytest.mark.parametrize("over,expect", [
    (dict(k=None), xb.ERR_NULL),
    (dict(packed=None), xb.ERR_NULL),
    (dict(f_pre=FAKE + 4), xb.ERR_ALIGN),
    (dict(packed=FAKE + 8), xb.ERR_ALIGN),
    (dict(fg=3), xb.ERR_DTYPE),
    (dict(dt=xb.BF16, chunk=32), xb.ERR_CHUNK),
    (dict(DH=24), xb.ERR_SHAPE),
    (dict(S=-1), xb.ERR_SHAPE),
    (dict(workspace_bytes=64), xb.ERR_WORKSPACE),
    (dict(B=0), xb.OK),
])
def test_seg_state_rejects_bad_arguments_before_device_work(over, expect):
    assert _seg_state(**over) == expect


def _combine(**over):
    a = dict(parts=FAKE, count=2, C0=None, n0=None, m0=None, C_out=FAKE, n_out=FAKE, m_out=FAKE,
             B=1, NH=2, DH=64, stream=None)
    a.update(over)
    return xb.xlstm_mlstm_state_combine(**a)


@pytest.mark.parametrize("over,expect", [
    (dict(parts=None), xb.ERR_NULL),
    (dict(C_out=None), xb.ERR_NULL),
    (dict(m_out=None), xb.ERR_NULL),
    (dict(count=-1), xb.ERR_SHAPE),
    (dict(DH=520), xb.ERR_SHAPE),
    (dict(n0=FAKE + 4), xb.ERR_ALIGN),
    (dict(C0=FAKE, C_out=FAKE), xb.ERR_UNSUPPORTED),       # in place is refused
    (dict(m0=FAKE + 64, m_out=FAKE + 64), xb.ERR_UNSUPPORTED),
    (dict(NH=0), xb.OK),
])
def test_state_combine_rejects_bad_arguments_before_device_work(over, expect):
    assert _combine(**over) == expect


def test_seg_state_sizes():
    # packed summary: C' [BH,DH,DH] + n' [BH,DH] + mloc, F [BH], padded to 4 floats
    assert xb.xlstm_mlstm_seg_state_floats(1, 8, 256) == (xb.OK, 8 * (256 * 256 + 256 + 2))
    assert xb.xlstm_mlstm_seg_state_floats(1, 1, 16) == (xb.OK, 276)      # 274 -> 276
    assert xb.xlstm_mlstm_seg_state_floats(1, 1, 20)[0] == xb.ERR_SHAPE
    # every segment summarised: at least the forward's workspace, plus one slot
    for dt, DH, L in ((xb.BF16, 256, 64), (xb.BF16, 64, 128), (xb.F32, 32, 16)):
        st, ws = xb.xlstm_mlstm_seg_state_workspace_size(1, 8, 4096, DH, L, dt)
        st2, wf = xb.xlstm_mlstm_fwd_workspace_size(1, 8, 4096, DH, L, dt)
        assert st == st2 == xb.OK and ws >= wf + 8 * (DH * DH + DH) * 4
    assert xb.xlstm_mlstm_seg_state_workspace_size(1, 8, 0, 64, 64, xb.BF16) == (xb.OK, 0)
