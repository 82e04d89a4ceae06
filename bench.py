"""Benchmark of the mLSTM cell forward and decode step on B200.

Default run (N = 1): the long-context forward (B=1, NH=8, S=16384, DH=256,
bf16 q/k/v, fp32 gates and state) is the timed step; one step is one full
forward over that batch (gate prologue, segment summaries, chunkwise outputs
and final state).  The decode step workload (B=256, NH=8, DH=512, fp32 state,
1024 consecutive tokens after a 512-token prefill) is timed in the same run and
reported under "decode", and the block epilogue after the cell (per-head
GroupNorm, learnable skip, external output gate) on the forward's shape under
"epilogue".  Inputs are seeded synthetic tensors of those shapes.

Under torchrun (N > 1) every rank runs its own replica of the same workload on
its own GPU (heads are independent, so the batch shards with no collective);
the timed region is bracketed by barriers and device syncs and the max over
ranks is reported.  ``--impl reference`` times the float64 CPU oracle instead
(rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_rnn_mlstm_b200 import binding as xb  # noqa: E402
from linear_rnn_mlstm_b200 import replicas  # noqa: E402
from linear_rnn_mlstm_b200 import synthetic as syn  # noqa: E402

METRIC = "mLSTM fwd tokens/s & % bf16 TC peak; decode-step HBM GB/s vs peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def fwd_flops(BH, S, DH, L):
    """Useful flops of the chunkwise forward: inter retrieval and state update
    (2*DH^2 each per token) and the causal-exact intra part ((L+1)*DH each for
    scores and values per token on average)."""
    return BH * S * (4.0 * DH * DH + 2.0 * (L + 1) * DH)


def fwd_token_bytes(DH, qkv_bytes):
    """Algorithmic HBM bytes per token: q, k, v, h in the q dtype, otilde fp32
    per element, itilde and ftilde fp32."""
    return 4 * DH * qkv_bytes + 4 * DH + 8


def state_bytes(BH, DH):
    return BH * 4 * (DH * DH + DH + 1)


def kernel_algorithmic_bytes(name, w, plan):
    """Bytes a launch of kernel `name` must move over one forward of `w`."""
    BH, S, DH = w.B * w.NH, w.S, w.DH
    qb = 2 if w.dtype == "bf16" else 4
    if name.startswith("segment_output"):
        return BH * S * fwd_token_bytes(DH, qb) + state_bytes(BH, DH)
    if name.startswith("segment_summary"):
        seg_tokens = BH * S * (plan["P"] - 1) / max(plan["P"], 1)
        return seg_tokens * (2 * DH * qb + 8) + BH * (plan["P"] - 1) * 4 * (DH * DH + DH)
    if name == "gate_prologue":
        return BH * S * 12
    return None


def source_sha(kernel):
    """sha1 of the source files a kernel is built from (the tensor-core kernels
    also depend on the tcgen05/TMA wrappers)."""
    files = {"segment_output_simt": ["fwd_simt.cu"], "segment_summary_simt": ["fwd_simt.cu"],
             "gate_prologue": ["fwd_simt.cu"], "step_rows": ["step.cu"], "step_state": ["step.cu"],
             "headnorm_gate": ["headnorm.cu"], "segment_output_rs": ["fwd_rs.cu", "tc_ptx.cuh"],
             "combine_keysplit": ["fwd_rs.cu"]}
    fns = files.get(kernel)
    if fns is None and kernel.endswith("_tc"):
        fns = ["fwd_tc.cu", "tc_ptx.cuh"]
    if fns is None:
        return None
    h = hashlib.sha1()
    for fn in fns:
        with open(os.path.join(ROOT, "linear_rnn_mlstm_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(kernel, units):
    """DRAM bytes per launch from the committed ncu summary, scaled to `units`
    processed, if the kernel source is unchanged since the capture; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except Exception:
        return None
    if not rec or rec.get("source_sha") != source_sha(kernel):
        return None
    return rec["dram_bytes_per_unit"] * units


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 7:
                self.samples.append(parts)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in self.samples:
            try:
                sm.append(float(p[0]))
                mx = float(p[1])
            except ValueError:
                continue
            for nm, val in zip(names, p[3:]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def physical_gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        items = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(items):
            return items[local_rank]
    return str(local_rank)


# ------------------------------------------------------------ oracle (CPU)
def cpu_baseline(w, max_tokens_per_head):
    """The float64 oracle as it stands, on a bounded sample of workload `w`:
    all heads, the first `max_tokens_per_head` tokens of each.  Returns the
    baseline record (tokens/s)."""
    import oracle
    S = min(w.S, max_tokens_per_head)
    inp = syn.fwd_inputs(w)
    sub = {k: v[:, :, :S] for k, v in inp.items()}
    t0 = time.perf_counter()
    oracle.fwd(sub["q"], sub["k"], sub["v"], sub["i_pre"], sub["f_pre"], sub["o_pre"], w.fgate)
    dt = time.perf_counter() - t0
    toks = w.B * w.NH * S
    cores = min(oracle.max_threads(), w.B * w.NH)
    return {"value": toks / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{w.B * w.NH} heads x first {S} tokens of the {w.name} workload "
                      f"({toks} tokens, {dt:.2f} s wall)"}


def run_reference(args):
    if not replicas.rank_env().reports:      # under torchrun only rank 0 runs the oracle
        return 0
    import oracle
    w = syn.WORKLOADS[args.config]
    S = min(w.S, args.ref_tokens)
    inp = syn.fwd_inputs(w)
    sub = {k: v[:, :, :S] for k, v in inp.items()}
    run = lambda: oracle.fwd(sub["q"], sub["k"], sub["v"], sub["i_pre"], sub["f_pre"],
                             sub["o_pre"], w.fgate)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = (time.perf_counter() - t0) / args.steps
    toks = w.B * w.NH * S
    value = toks / dt
    cores = min(oracle.max_threads(), w.B * w.NH)
    sample = f"{w.B * w.NH} heads x first {S} tokens of the {w.name} workload per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.chunk, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, chunk, n):
    return {"workload": f"{w.name} mLSTM fwd: B={w.B} NH={w.NH} S={w.S} DH={w.DH} {w.dtype} q/k/v, "
                        f"{w.fgate} forget gate, chunk {chunk}",
            "B": w.B, "NH": w.NH, "S": w.S, "DH": w.DH, "chunk": chunk,
            "global_batch": w.B * n, "seq_len": w.S, "parallelism": f"replicas x{n} (heads independent)"}


# ----------------------------------------------------------------- GPU arm
def make_fwd_runner(x, w, chunk, dev, path):
    BH = w.B * w.NH
    h = torch.empty_like(x["q"])
    C = torch.empty((w.B, w.NH, w.DH, w.DH), dtype=torch.float32, device=dev)
    n = torch.empty((w.B, w.NH, w.DH), dtype=torch.float32, device=dev)
    m = torch.empty((w.B, w.NH), dtype=torch.float32, device=dev)
    dt = xb.BF16 if w.dtype == "bf16" else xb.F32
    fg = xb.FGATE_EXP if w.fgate == "exp" else xb.FGATE_SIGMOID
    st, nbytes = xb.xlstm_mlstm_fwd_workspace_size(w.B, w.NH, w.S, w.DH, chunk, dt, path)
    assert st == xb.OK, xb.status_string(st)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    ptrs = [x[k].data_ptr() for k in ("q", "k", "v", "i_pre", "f_pre", "o_pre")]

    def run():
        s = xb.xlstm_mlstm_fwd(*ptrs, h.data_ptr(), None, None, None, C.data_ptr(), n.data_ptr(),
                               m.data_ptr(), w.B, w.NH, w.S, w.DH, chunk, dt, fg, ws.data_ptr(),
                               ws.numel(), stream, path)
        if s != xb.OK:
            raise xb.XlstmError(s, "xlstm_mlstm_fwd")
    return run, (h, C, n, m), BH


def time_region(fn, steps, env, dev):
    """Device time of `steps` calls, between a barrier and a synchronize on both
    sides; the max over ranks (every rank gets it)."""
    replicas.barrier(env)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize(dev)
    replicas.barrier(env)
    return replicas.max_over_ranks(e0.elapsed_time(e1), env, dev)


def plan_info(w, chunk, path):
    # segments chosen by the library: recover P from the workspace size
    BH, DH = w.B * w.NH, w.DH
    dt = xb.BF16 if w.dtype == "bf16" else xb.F32
    _, base = xb.xlstm_mlstm_fwd_workspace_size(w.B, w.NH, w.S, DH, chunk, dt, path, 1)
    _, auto = xb.xlstm_mlstm_fwd_workspace_size(w.B, w.NH, w.S, DH, chunk, dt, path, 0)
    per_seg = BH * (DH * DH + DH) * 4
    P = 1 + max(0, round((auto - base) / per_seg))
    return {"P": P}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="long", choices=sorted(syn.WORKLOADS))
    ap.add_argument("--chunk", type=int, default=64)
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tensor", "tensor_tmem", "tensor_rs"])
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--decode-B", type=int, default=0,
                    help="batch of the decode workload (0 = its full B of 256); profiling only")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-epilogue", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-slstm", action="store_true")
    ap.add_argument("--skip-backward", action="store_true")
    ap.add_argument("--skip-seqpar", action="store_true")
    ap.add_argument("--skip-sweep", action="store_true",
                    help="skip the per-config / per-chunk entries (small, block, long at 128 and 256)")
    ap.add_argument("--ref-tokens", type=int, default=4096,
                    help="tokens per head in each reference (oracle) step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    env = replicas.rank_env()
    world, rank, local_rank = env.world, env.rank, env.local_rank
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    replicas.init(env, "nccl", dev, timeout_s=300)
    xb.load()
    peaks, peak_src = load_peaks()
    path = {"auto": xb.PATH_AUTO, "simt": xb.PATH_SIMT, "tensor": xb.PATH_TENSOR,
            "tensor_tmem": xb.PATH_TENSOR_TMEM, "tensor_rs": xb.PATH_TENSOR_RS}[args.path]

    # ------------------------------------------------------------ forward
    w = syn.WORKLOADS[args.config]
    inp = syn.fwd_inputs(w, seed=replicas.replica_seed(w.seed, rank))
    x = {k: v.to(dev).contiguous() for k, v in inp.items()}
    run, outs, BH = make_fwd_runner(x, w, args.chunk, dev, path)
    sampler = ClockSampler(physical_gpu_index(local_rank)) if rank == 0 else None
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize(dev)
    # the step time is taken without per-kernel events (they would stand between
    # the chained launches); a second pass of the same steps gives the breakdown
    ms = time_region(run, args.steps, env, dev)
    xb.xlstm_profile_begin()
    time_region(run, args.steps, env, dev)
    _, kt = xb.xlstm_profile_end()
    ms_step = ms / args.steps
    tokens = w.B * w.NH * w.S
    value = replicas.job_throughput(tokens, env, ms_step * 1e-3)
    launches = sum(v[0] for v in kt.values())
    kernels = {k: {"launches": v[0], "avg_us": 1e3 * v[1] / max(v[0], 1),
                   "share": v[1] / max(sum(u[1] for u in kt.values()), 1e-12)}
               for k, v in kt.items()}
    top = max(kt.items(), key=lambda kv: kv[1][1])[0] if kt else None
    plan = plan_info(w, args.chunk, path)
    alg = kernel_algorithmic_bytes(top, w, plan) if top else None
    top_us = kernels[top]["avg_us"] if top else None
    roofline = None
    if alg:
        achieved = alg / (top_us * 1e-6) / 1e9
        roofline = {"kernel": top, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                    "traffic": ncu_traffic(top, BH * w.S), "algorithmic_bytes": alg,
                    "peak_source": f"{peak_src} (burst copy)"}
    flops = fwd_flops(BH, w.S, w.DH, args.chunk)
    tflops = flops / (ms_step * 1e-3) / 1e12
    tc = {"useful_tflops": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
          "frac": tflops / peaks["bf16_tflops"], "useful_flops_per_step": flops,
          "peak_source": f"{peak_src} (burst cuBLAS bf16)"}
    step_bytes = tokens * fwd_token_bytes(w.DH, 2 if w.dtype == "bf16" else 4) + state_bytes(BH, w.DH)
    whole = {"achieved_gbs": step_bytes / (ms_step * 1e-3) / 1e9,
             "frac": step_bytes / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"],
             "algorithmic_bytes_per_step": step_bytes}

    # ------------------------------------------------------------- end to end
    e2e = None
    if not args.skip_e2e:
        e2e = run_e2e(args, w, inp, x, outs, run, dev, env, path)
    del x, outs, run

    # -------------------------------------------------- block epilogue (next row)
    epilogue = None
    if not args.skip_epilogue:
        epilogue = run_epilogue(args, w, dev, env, peaks, peak_src)

    # ------------------------------------------------------ sLSTM (next row)
    slstm = None
    if not args.skip_slstm:
        slstm = run_slstm(args, dev, env, with_cpu=(rank == 0 and world == 1 and not args.skip_cpu))

    # --------------------------------------------------- backward (next row)
    backward = None
    if not args.skip_backward:
        backward = run_backward(args, dev, env, peaks, peak_src)

    # ------------------------------------- sequence parallelism (next row)
    seqpar_entry = None
    if not args.skip_seqpar:
        seqpar_entry = run_seqpar(args, dev, env)

    # ----------------------------------------------------------------- decode
    decode = None
    if not args.skip_decode:
        decode = run_decode(args, dev, env, peaks, peak_src)

    # ------------------------------------------- every config and chunk size
    sweep = None
    if not args.skip_sweep:
        sweep = run_sweep(args, dev, env, peaks, peak_src, with_cpu=(rank == 0 and world == 1 and not args.skip_cpu))

    clocks = sampler.stop() if sampler else None

    # ------------------------------------------------------------ CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        cpu = cpu_baseline(w, w.S)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if (w.dtype == "bf16" and any(k.endswith(("_tc", "_rs")) for k in kt)) else "f32",
                "data": "synthetic (seeded N(0,1)-based draws of the workload shapes)",
                "config": dict(workload_config(w, args.chunk, world),
                               l2="inputs 406 MB > 126 MB L2; no flush" if w.name == "long"
                               else "inputs may fit L2", segments=plan["P"],
                               path=args.path),
                "roofline": roofline, "tc": tc, "hbm_whole_step": whole,
                "kernels": kernels, "gpu_launches": launches, "cpu_baseline": cpu, "e2e": e2e,
                "clocks": clocks, "decode": decode, "epilogue": epilogue, "slstm": slstm, "backward": backward,
                "sequence_parallel": seqpar_entry,
                "sweep": sweep}
        print(json.dumps(line), flush=True)
    replicas.barrier(env)
    replicas.shutdown(env)
    return 0


SWEEP = (("small", 64), ("block", 64), ("block", 128), ("long", 128), ("long", 256))
SWEEP_CPU_TOKENS = {"small": 1024, "block": 256, "long": 1024}


def path_name(w, chunk):
    st, fam = xb.xlstm_mlstm_fwd_path(w.DH, chunk, xb.BF16 if w.dtype == "bf16" else xb.F32)
    return {xb.PATH_TENSOR: "tensor (tcgen05)", xb.PATH_SIMT: "simt (fp32 CUDA cores)"}.get(fam, str(fam))


def run_sweep(args, dev, env, peaks, peak_src, with_cpu):
    """The other forward configurations and chunk sizes, each timed on its own
    (AUTO path, which kernel family ran is named): per step, the L2 is flushed
    by writing a 256 MB buffer outside the timed events, then one forward is
    timed with CUDA events; the median over the steps is reported.  Each entry
    carries tokens/s, useful TFLOP/s, the whole-step HBM fraction, the dominant
    kernel's roofline and the float64 oracle on a bounded sample beside it."""
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    out = []
    for name, chunk in SWEEP:
        w = syn.WORKLOADS[name]
        inp = syn.fwd_inputs(w, seed=replicas.replica_seed(w.seed, env.rank))
        x = {k: v.to(dev).contiguous() for k, v in inp.items()}
        run, outs, BH = make_fwd_runner(x, w, chunk, dev, xb.PATH_AUTO)
        for _ in range(3):
            run()
        torch.cuda.synchronize(dev)
        steps = max(5, min(args.steps, 10))
        times = []
        for profiled in (False, True):      # step times without per-kernel events, then the breakdown
            if profiled:
                xb.xlstm_profile_begin()
            for _ in range(steps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                run()
                e1.record()
                torch.cuda.synchronize(dev)
                if not profiled:
                    times.append(e0.elapsed_time(e1))
        _, kt = xb.xlstm_profile_end()
        ms = replicas.max_over_ranks(statistics.median(times), env, dev)
        tokens = w.B * w.NH * w.S
        eb = 2 if w.dtype == "bf16" else 4
        step_bytes = tokens * fwd_token_bytes(w.DH, eb) + state_bytes(BH, w.DH)
        flops = fwd_flops(BH, w.S, w.DH, chunk)
        kernels = {k: {"launches": v[0], "avg_us": 1e3 * v[1] / max(v[0], 1)} for k, v in kt.items()}
        top = max(kt.items(), key=lambda kv: kv[1][1])[0] if kt else None
        roof = None
        if top:
            alg = kernel_algorithmic_bytes(top, w, plan_info(w, chunk, xb.PATH_AUTO))
            if alg:
                ach = alg / (kernels[top]["avg_us"] * 1e-6) / 1e9
                roof = {"kernel": top, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": ach / peaks["hbm_gbs"], "algorithmic_bytes": alg,
                        "note": "kernel average over the flushed steps"}
        entry = {"workload": workload_config(w, chunk, env.world)["workload"], "chunk": chunk,
                 "path": path_name(w, chunk), "ms_per_step": ms,
                 "tokens_per_s": replicas.job_throughput(tokens, env, ms * 1e-3),
                 "useful_tflops": flops / (ms * 1e-3) / 1e12,
                 "tc_frac": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                 "hbm_frac_whole_step": step_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                 "algorithmic_bytes_per_step": step_bytes, "useful_flops_per_step": flops,
                 "l2": "256 MB flush before every timed step", "roofline": roof, "kernels": kernels,
                 "peak_source": f"{peak_src} (burst copy / burst cuBLAS bf16)"}
        if with_cpu:
            entry["cpu_baseline"] = cpu_baseline(w, SWEEP_CPU_TOKENS[name])
        out.append(entry)
        del x, outs, run
    del flush
    return out


def run_e2e(args, w, inp, x, outs, run, dev, env, path):
    """End to end through the C ABI with host buffers: every step copies that
    step's inputs from pinned host memory to the device, runs the forward and
    copies h and the final state back.  Steps are pipelined over two device
    buffer sets and three streams (upload, compute, download), so the upload
    of step k+1 and the download of step k-1 overlap the forward of step k
    (PCIe is full duplex); every copy of every timed step is inside the timed
    region, which ends when the last download has landed."""
    pin = {k: v.pin_memory() for k, v in inp.items()}
    x2 = {k: torch.empty_like(v) for k, v in x.items()}
    run2, outs2, _ = make_fwd_runner(x2, w, args.chunk, dev, path)
    bufs = [(x, outs, run), (x2, outs2, run2)]
    hosts = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs] for _ in range(2)]
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_comp + ev_out:
        e.record(comp)
    state = {"k": 0}

    def step():
        k = state["k"]
        state["k"] += 1
        b = k % 2
        xin, yout, fn = bufs[b]
        with torch.cuda.stream(up):
            up.wait_event(ev_comp[b])                 # the forward that last read these inputs
            for name in xin:
                xin[name].copy_(pin[name], non_blocking=True)
            ev_in[b].record(up)
        comp.wait_event(ev_in[b])
        comp.wait_event(ev_out[b])                    # the download that last read these outputs
        fn()
        ev_comp[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(ev_comp[b])
            for hst, dv in zip(hosts[b], yout):
                hst.copy_(dv, non_blocking=True)
            ev_out[b].record(down)

    def drain():
        comp.wait_event(ev_out[0])
        comp.wait_event(ev_out[1])

    for _ in range(2):
        step()
    drain()
    torch.cuda.synchronize(dev)
    steps = max(3, min(args.steps, 10))

    def timed():
        step()
    replicas.barrier(env)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for _ in range(steps):
        timed()
    drain()
    e1.record(comp)
    torch.cuda.synchronize(dev)
    replicas.barrier(env)
    ms_e2e = replicas.max_over_ranks(e0.elapsed_time(e1), env, dev) / steps
    tokens = w.B * w.NH * w.S
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in hosts[0])
    del x2, outs2, run2
    return {"value": replicas.job_throughput(tokens, env, ms_e2e * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "upload, forward, download on three streams over two buffer sets"}


def run_epilogue(args, w, dev, env, peaks, peak_src):
    """The mLSTM block's epilogue after the cell (per-head GroupNorm, learnable
    skip, SiLU external output gate) on the forward workload's shape, timed
    alone: h [B,NH,S,DH] -> y [B,S,NH*DH]."""
    B, NH, S, DH = w.B, w.NH, w.S, w.DH
    inp = syn.epilogue_inputs(B, NH, S, DH, w.dtype, seed=replicas.replica_seed(w.seed, env.rank))
    x = {k: v.to(dev).contiguous() for k, v in inp.items()}
    y = torch.empty(x["x_skip"].shape, dtype=x["h"].dtype, device=dev)
    dt = xb.BF16 if w.dtype == "bf16" else xb.F32
    stream = torch.cuda.current_stream(dev).cuda_stream
    ptrs = [x[k].data_ptr() for k in ("h", "gamma", "beta", "skip_w", "x_skip", "z")]

    def one():
        st = xb.xlstm_mlstm_headnorm_gate(*ptrs, y.data_ptr(), B, NH, S, DH, 1e-5, dt,
                                          xb.OGATE_SILU, stream)
        if st != xb.OK:
            raise xb.XlstmError(st, "xlstm_mlstm_headnorm_gate")
    for _ in range(max(3, args.warmup)):
        one()
    torch.cuda.synchronize(dev)
    steps = max(10, args.steps)
    xb.xlstm_profile_begin()
    ms = time_region(one, steps, env, dev)
    _, kt = xb.xlstm_profile_end()
    rows = B * S * NH
    eb = 2 if w.dtype == "bf16" else 4
    alg = rows * DH * 4 * eb + 3 * 4 * NH * DH         # h, x_skip, z in; y out; 3 parameter rows
    k = kt.get("headnorm_gate", (0, 0.0))
    us = 1e3 * k[1] / max(k[0], 1)
    ach = alg / (us * 1e-6) / 1e9 if us > 0 else None
    return {"kernel": "headnorm_gate", "us_per_launch": us, "ms_per_call": ms / steps,
            "launches": k[0],
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": (ach / peaks["hbm_gbs"]) if ach else None,
                         "traffic": ncu_traffic("headnorm_gate", rows), "algorithmic_bytes": alg,
                         "peak_source": f"{peak_src} (burst copy)"},
            "config": f"block epilogue: h [{B},{NH},{S},{DH}] {w.dtype} -> y [{B},{S},{NH * DH}], "
                      f"skip on, SiLU gate, eps 1e-5; {alg / 1e6:.0f} MB per launch (> L2)"}


def run_slstm(args, dev, env, with_cpu):
    """The sLSTM forward on its timing workload (B4 NH4 S2048 DH256, fp32): one
    call walks the sequence; tokens/s and microseconds per recurrent step, with
    the float64 sLSTM oracle on a bounded sample beside it."""
    c = syn.SLSTM
    B, NH, S, DH = c["B"], c["NH"], c["S"], c["DH"]
    inp = syn.slstm_inputs(B, NH, S, DH, seed=replicas.replica_seed(11, env.rank))
    x = {k: v.to(dev).contiguous() for k, v in inp.items()}
    run = lambda: xb.slstm_fwd(x["zx"], x["ix"], x["fx"], x["ox"], x["R"], "sigmoid")
    for _ in range(max(3, args.warmup)):
        run()
    torch.cuda.synchronize(dev)
    steps = max(3, min(args.steps, 10))
    ms = time_region(run, steps, env, dev) / steps
    xb.xlstm_profile_begin()
    run()
    torch.cuda.synchronize(dev)
    _, kt = xb.xlstm_profile_end()
    tokens = B * NH * S
    out = {"metric": "sLSTM fwd tokens/s", "value": replicas.job_throughput(tokens, env, ms * 1e-3),
           "unit": "tokens/s", "ms_per_call": ms, "us_per_step": 1e3 * ms / S,
           "kernels": {k: {"launches": v[0], "avg_us": 1e3 * v[1] / max(v[0], 1)} for k, v in kt.items()},
           "config": f"sLSTM fwd: B={B} NH={NH} S={S} DH={DH} fp32, sigmoid forget gate, zero initial state; "
                     f"{B * NH} heads walk their sequences concurrently"}
    if with_cpu:
        import oracle.slstm as so
        Ss = S                                       # the whole workload: ~0.3 s of float64
        sub = {k: (v[:, :, :Ss] if k != "R" else v).numpy() for k, v in inp.items()}
        t0 = time.perf_counter()
        so.fwd(sub["zx"], sub["ix"], sub["fx"], sub["ox"], sub["R"], "sigmoid")
        dt = time.perf_counter() - t0
        import oracle
        out["cpu_baseline"] = {"value": B * NH * Ss / dt, "unit": "tokens/s",
                               "cores": min(oracle.max_threads(), B * NH), "kind": "oracle",
                               "sample": f"{B * NH} heads x first {Ss} steps ({B * NH * Ss} tokens, {dt:.2f} s wall)"}
    return out


def run_backward(args, dev, env, peaks, peak_src):
    """The backward (fp32 kernels) on the small workload and on the long one,
    chunk 64, gradients of sum(dh h) with dh ~ N(0, 1) in bf16: time per call
    and HBM fraction at the algorithmic 22 DH + 16 bytes per token (bf16 q, k,
    v, dh in and dq, dk, dv out; fp32 o in and do out; the gates and their
    gradients)."""
    out = []
    for name in ("small", "long"):
        w = syn.WORKLOADS[name]
        inp = syn.fwd_inputs(w, seed=replicas.replica_seed(w.seed, env.rank))
        x = {k: v.to(dev).contiguous() for k, v in inp.items()}
        g = torch.Generator().manual_seed(5)
        dh = torch.randn(inp["q"].shape, generator=g).to(inp["q"].dtype).to(dev)
        run = lambda: xb.mlstm_bwd(x["q"], x["k"], x["v"], x["i_pre"], x["f_pre"], x["o_pre"], dh,
                                   chunk=64, fgate=w.fgate)
        run()
        torch.cuda.synchronize(dev)
        steps = 3
        ms = time_region(run, steps, env, dev) / steps
        xb.xlstm_profile_begin()
        run()
        torch.cuda.synchronize(dev)
        _, kt = xb.xlstm_profile_end()
        tokens = w.B * w.NH * w.S
        alg = tokens * (22 * w.DH + 16)
        ach = alg / (ms * 1e-3) / 1e9
        out.append({"workload": f"{name}: B={w.B} NH={w.NH} S={w.S} DH={w.DH} {w.dtype}, chunk 64",
                    "ms_per_call": ms, "tokens_per_s": replicas.job_throughput(tokens, env, ms * 1e-3),
                    "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                 "frac": ach / peaks["hbm_gbs"], "algorithmic_bytes": alg,
                                 "peak_source": f"{peak_src} (burst copy)"},
                    "kernels": {k: {"launches": v[0], "avg_us": 1e3 * v[1] / max(v[0], 1)}
                                for k, v in kt.items()}})
        del x, dh
    return out


def run_seqpar(args, dev, env):
    """Sequence parallelism on the long workload (B1 NH8 S16384 DH256 bf16, chunk
    64): the one sequence cut into as many slices as there are ranks, each rank
    summarising its slice, one all-gather of the summaries, a fold, and the
    slice's forward (seqpar.sequence_parallel_fwd); time = max over ranks,
    tokens/s over the whole sequence (strong scaling).  Beside it, measured on
    this GPU, what each rank of an eight-way split runs: the summary of a
    2048-token slice, the fold of seven summaries, and the slice's forward from
    a folded state."""
    from linear_rnn_mlstm_b200 import seqpar
    w = syn.LONG
    chunk = 64
    world, rank = env.world, env.rank
    inp = syn.fwd_inputs(w, seed=w.seed)             # every rank draws the same sequence
    a, b = rank * w.S // world, (rank + 1) * w.S // world
    x = {k: v[:, :, a:b].to(dev).contiguous() for k, v in inp.items()}
    args_fwd = [x[k] for k in ("q", "k", "v", "i_pre", "f_pre", "o_pre")]
    run = lambda: seqpar.sequence_parallel_fwd(*args_fwd, chunk=chunk, fgate=w.fgate)
    for _ in range(max(3, args.warmup)):
        run()
    torch.cuda.synchronize(dev)
    steps = max(3, min(args.steps, 10))
    ms = time_region(run, steps, env, dev) / steps
    tokens = w.B * w.NH * w.S
    out = {"metric": "mLSTM fwd tokens/s, one sequence split over the ranks",
           "value": tokens / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "n_ranks": world,
           "scaling": "strong", "tokens_per_rank": w.B * w.NH * (b - a),
           "config": f"long: B={w.B} NH={w.NH} S={w.S} DH={w.DH} bf16, chunk {chunk}, "
                     f"S split into {world} slice(s)"}
    del x, args_fwd
    # one rank's share of an eight-way split, timed alone on this GPU
    R = 8
    Ss = w.S // R
    sl = {k: v[:, :, :Ss].to(dev).contiguous() for k, v in inp.items()}
    nf = xb.seg_state_floats(w.B, w.NH, w.DH)
    parts = torch.zeros((R, nf), dtype=torch.float32, device=dev)
    for r in range(R):
        xb.mlstm_seg_state(sl["k"], sl["v"], sl["i_pre"], sl["f_pre"], chunk=chunk, fgate=w.fgate,
                           packed=parts[r])
    C, n, m = xb.mlstm_state_combine(parts, R - 1, w.B, w.NH, w.DH)
    pieces = {
        "seg_state": lambda: xb.mlstm_seg_state(sl["k"], sl["v"], sl["i_pre"], sl["f_pre"], chunk=chunk,
                                                fgate=w.fgate, packed=parts[0]),
        "state_combine_7": lambda: xb.mlstm_state_combine(parts, R - 1, w.B, w.NH, w.DH, out=(C, n, m)),
        "fwd_from_state": lambda: xb.mlstm_fwd(*(sl[k] for k in ("q", "k", "v", "i_pre", "f_pre", "o_pre")),
                                               chunk=chunk, fgate=w.fgate, C0=C, n0=n, m0=m),
    }
    share = {}
    for name, fn in pieces.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        share[name + "_ms"] = time_region(fn, 10, env, dev) / 10
    share["summary_bytes_per_rank"] = nf * 4
    out["eight_way_rank_share"] = dict(share, slice_tokens=w.B * w.NH * Ss,
                                       note="per-rank device time of an 8-GPU split (exchange of "
                                            f"{R} x {nf * 4 / 1e6:.1f} MB not included)")
    return out


def run_decode(args, dev, env, peaks, peak_src):
    rank, world = env.rank, env.world
    d = syn.DECODE
    if args.decode_B:
        import dataclasses
        d = dataclasses.replace(d, B=args.decode_B)
    T = args.decode_steps
    BH, DH = d.B * d.NH, d.DH
    pre = syn.fwd_inputs(d.prefill(), seed=replicas.replica_seed(d.seed, rank))
    x = {k: v.to(dev) for k, v in pre.items()}
    _, C, n, m = xb.mlstm_fwd(x["q"], x["k"], x["v"], x["i_pre"], x["f_pre"], x["o_pre"],
                              chunk=d.prefill_chunk, fgate=d.fgate)
    del x
    steps = []
    for t in range(T):
        s = syn.step_inputs(d, t, seed=replicas.replica_seed(d.seed, rank))
        steps.append({k: v.to(dev, non_blocking=False) for k, v in s.items()})
    h = torch.empty((d.B, d.NH, DH), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    fg = xb.FGATE_EXP if d.fgate == "exp" else xb.FGATE_SIGMOID
    cur = [0]

    def one():
        s = steps[cur[0] % T]
        cur[0] += 1
        st = xb.xlstm_mlstm_step(s["q"].data_ptr(), s["k"].data_ptr(), s["v"].data_ptr(),
                                 s["i_pre"].data_ptr(), s["f_pre"].data_ptr(), s["o_pre"].data_ptr(),
                                 h.data_ptr(), C.data_ptr(), n.data_ptr(), m.data_ptr(),
                                 d.B, d.NH, DH, xb.BF16, fg, stream)
        if st != xb.OK:
            raise xb.XlstmError(st, "xlstm_mlstm_step")
    for _ in range(max(3, args.warmup)):
        one()
    torch.cuda.synchronize(dev)
    cur[0] = 0
    xb.xlstm_profile_begin()
    ms = time_region(one, T, env, dev)
    _, kt = xb.xlstm_profile_end()
    ms_step = ms / T
    step_bytes = BH * (8.0 * DH * DH + 8 * DH + 8) + BH * DH * (3 * 2 + 4 + 2) + BH * 8
    gbs = step_bytes / (ms_step * 1e-3) / 1e9
    rows = kt.get("step_rows", (0, 0.0))
    rows_us = 1e3 * rows[1] / max(rows[0], 1)
    row_bytes = BH * (8.0 * DH * DH) + BH * DH * (3 * 2 + 4 + 2 + 4) + BH * 12
    ach = row_bytes / (rows_us * 1e-6) / 1e9 if rows_us > 0 else None
    return {"metric": "decode-step HBM GB/s", "value": gbs * world, "unit": "GB/s",
            "per_gpu_frac": gbs / peaks["hbm_gbs"], "ms_per_step": ms_step, "steps": T,
            "tokens_per_s": replicas.job_throughput(BH, env, ms_step * 1e-3),
            "algorithmic_bytes_per_step": step_bytes,
            "roofline": {"kernel": "step_rows", "bound": "hbm", "achieved": ach,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": (ach / peaks["hbm_gbs"]) if ach else None,
                         "traffic": ncu_traffic("step_rows", BH), "peak_source": f"{peak_src} (burst copy)"},
            "kernels": {k: {"launches": v[0], "avg_us": 1e3 * v[1] / max(v[0], 1)} for k, v in kt.items()},
            "gpu_launches": sum(v[0] for v in kt.values()),
            "config": f"decode: B={d.B} NH={d.NH} DH={DH} bf16 q/k/v, fp32 state (2 GiB, > L2), "
                      f"prefill S={d.prefill_S} chunk {d.prefill_chunk}, {T} consecutive tokens"}


if __name__ == "__main__":
    sys.exit(main())
