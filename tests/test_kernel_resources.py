"""Register, spill and stack budgets of the kernels, from ptxas's resource
report (``nvcc -Xptxas -v``) on the CPU, so that an edit which makes a hot
kernel spill, or outgrow the register file at its launch width, fails here
before it reaches a GPU.  Compiles every ``csrc/*.cu`` with the library's own
flags (about a quarter of a minute, in parallel)."""
import concurrent.futures as cf
import glob
import os
import re
import subprocess

import pytest

from linear_rnn_mlstm_b200 import build as libbuild

REGISTER_FILE = 65536          # 32-bit registers per SM (and per CTA at most)
STACK_LIMIT = 1024             # default per-thread stack, bytes

# kernels on the forward / decode hot path: no spills allowed
HOT = ("segment_output_tc_kernel", "segment_summary_tc_kernel", "segment_scan_kernel",
       "gate_prologue_kernel", "step_stream_kernel", "step_rows_kernel", "step_state_kernel",
       "headnorm_gate_kernel", "combine_keysplit_kernel", "slstm_cluster_kernel", "state_mma_kernel",
       "state_fold_kernel", "state_walk_kernel", "token_fwd_tc_kernel",
       "token_grad_tc_kernel")
# threads per CTA the launchers use for the tensor-core and streamed kernels
LAUNCH_THREADS = {"segment_output_tc_kernel": 448, "segment_summary_tc_kernel": 320,
                  "slstm_cluster_kernel": 256, "state_mma_kernel": 128,
                  "state_walk_kernel": 384, "token_fwd_tc_kernel": 512, "token_grad_tc_kernel": 512}


def _ptxas_report(src):
    cmd = [libbuild.nvcc(), *libbuild.ARCH, *libbuild.NVCC_FLAGS, "-Xptxas", "-v", "-c", src,
           "-o", os.devnull]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    kernels, cur = {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
            kernels[cur] = {}
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads",
                      line)
        if m and cur:
            kernels[cur].update(stack=int(m.group(1)), spill=int(m.group(2)) + int(m.group(3)))
        m = re.search(r"Used (\d+) registers", line)
        if m and cur:
            kernels[cur]["regs"] = int(m.group(1))
    return kernels


@pytest.fixture(scope="module")
def report():
    srcs = sorted(glob.glob(os.path.join(libbuild.CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        parts = list(ex.map(_ptxas_report, srcs))
    out = {}
    for p in parts:
        out.update(p)
    return out


def _named(report, short):
    return {k: v for k, v in report.items() if short in k}


def test_every_hot_path_kernel_is_reported(report):
    for short in HOT:
        assert _named(report, short), f"no ptxas report for {short}"


def test_hot_path_kernels_do_not_spill(report):
    for short in HOT:
        for name, r in _named(report, short).items():
            assert r["spill"] == 0, f"{short}: {r['spill']} bytes of spills ({name})"


def test_stack_frames_fit_the_default_limit(report):
    for name, r in report.items():
        assert r["stack"] <= STACK_LIMIT, f"{name}: {r['stack']} bytes of stack"


def test_tensor_core_kernels_fit_the_register_file_at_their_launch_width(report):
    for short, threads in LAUNCH_THREADS.items():
        found = _named(report, short)
        assert found
        for name, r in found.items():
            assert r["regs"] * threads <= REGISTER_FILE, f"{short}: {r['regs']} x {threads}"
