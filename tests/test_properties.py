"""Properties of the GPU path that hold at any size (no oracle needed):
chunk-size invariance, segment-count invariance, split continuity of the
state (fwd(S) = fwd(S1) -> fwd(S2) = fwd(S-k) -> k steps; section 2.5 of the
paper: linear time, constant memory), and head/batch permutation
equivariance (section 2.3: no memory mixing across heads)."""
import numpy as np
import pytest
import torch

from linear_rnn_mlstm_b200 import binding as xb
from linear_rnn_mlstm_b200 import synthetic as syn

from parity import assert_close, errors, to_cuda

pytestmark = pytest.mark.gpu


def _fwd(x, chunk, fgate, path=xb.PATH_AUTO, segments=0, state=(None, None, None)):
    h, C, n, m = xb.mlstm_fwd(x["q"], x["k"], x["v"], x["i_pre"], x["f_pre"], x["o_pre"],
                              chunk=chunk, fgate=fgate, path=path, segments=segments,
                              C0=state[0], n0=state[1], m0=state[2])
    return h, C, n, m


def test_chunk_size_invariance_long_context_shape():
    w = syn.custom("inv", 1, 4, 4096, 256, syn.LONG, seed=2)
    x = to_cuda(syn.fwd_inputs(w))
    outs = {c: _fwd(x, c, w.fgate) for c in (64, 128, 256)}
    ref = outs[64][0].float().cpu().numpy()
    for c in (128, 256):
        assert_close(outs[c][0].float().cpu().numpy(), ref, "bf16", f"h chunk {c} vs 64")
        assert errors(outs[c][1].cpu().numpy(), outs[64][1].cpu().numpy())[1] <= 1e-2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_segment_count_invariance(dtype):
    w = syn.custom("seg", 2, 2, 1000, 64, syn.SMALL, dtype=dtype, seed=4)
    x = to_cuda(syn.fwd_inputs(w))
    ref = _fwd(x, 64, w.fgate, segments=1)
    for seg in (2, 5, 16):
        h, C, n, m = _fwd(x, 64, w.fgate, segments=seg)
        # two fp32 runs with different rounding paths over 1000 tokens: the
        # compounding bound of the wide-gate case applies, not the tiny one
        tol = "f32_wide" if dtype == "f32" else "bf16"
        assert_close(h.float().cpu().numpy(), ref[0].float().cpu().numpy(), tol)
        assert np.max(np.abs(m.cpu().numpy() - ref[3].cpu().numpy())) <= 1e-4


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_split_continuity(dtype):
    w = syn.custom("split", 2, 2, 640, 128, syn.SMALL, dtype=dtype, seed=6)
    x = to_cuda(syn.fwd_inputs(w))
    h, C, n, m = _fwd(x, 64, w.fgate)
    s1 = 384
    a = {k: v[:, :, :s1].contiguous() for k, v in x.items()}
    b = {k: v[:, :, s1:].contiguous() for k, v in x.items()}
    ha, Ca, na, ma = _fwd(a, 64, w.fgate)
    hb, Cb, nb, mb = _fwd(b, 64, w.fgate, state=(Ca, na, ma))
    tol = "f32_wide" if dtype == "f32" else "bf16"
    got = torch.cat([ha, hb], 2).float().cpu().numpy()
    assert_close(got, h.float().cpu().numpy(), tol)
    assert errors(Cb.cpu().numpy(), C.cpu().numpy())[1] <= (1e-5 if dtype == "f32" else 1e-2)
    # forward over S-k, then k decode steps
    k = 16
    hc, Cc, nc, mc = _fwd({kk: v[:, :, :640 - k].contiguous() for kk, v in x.items()}, 64, w.fgate)
    for t in range(640 - k, 640):
        y = {kk: v[:, :, t].contiguous() for kk, v in x.items()}
        ht = xb.mlstm_step(y["q"], y["k"], y["v"], y["i_pre"], y["f_pre"], y["o_pre"],
                           Cc, nc, mc, fgate=w.fgate)
        assert_close(ht.float().cpu().numpy(), h[:, :, t].float().cpu().numpy(), tol)
    assert errors(Cc.cpu().numpy(), C.cpu().numpy())[1] <= (1e-5 if dtype == "f32" else 1e-2)


def test_head_and_batch_permutation_equivariance():
    w = syn.custom("perm", 3, 4, 300, 64, syn.SMALL, seed=8)
    x = to_cuda(syn.fwd_inputs(w))
    h, C, n, m = _fwd(x, 64, w.fgate)
    pb = torch.tensor([2, 0, 1], device="cuda")
    ph = torch.tensor([3, 1, 0, 2], device="cuda")
    P = lambda t: t[pb][:, ph].contiguous()
    h2, C2, n2, m2 = _fwd({k: P(v) for k, v in x.items()}, 64, w.fgate)
    assert torch.equal(h2, P(h)) and torch.equal(C2, P(C)) and torch.equal(m2, P(m))
