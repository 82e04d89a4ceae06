"""The benchmark's command-line contract on the CPU: the reference arm (the
float64 oracle timed on the host) prints exactly one JSON line with every key
the result line needs, and too few warm-up steps are refused."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env=None):
    e = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        e.pop(k, None)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=e,
                          capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_one_complete_line():
    r = _bench("--impl", "reference", "--steps", "2", "--warmup", "3", "--ref-tokens", "64")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 3
    assert line["value"] > 0 and line["higher_is_better"] is True and line["unit"] == "tokens/s"
    assert line["config"]["workload"].startswith("long")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert "64 tokens" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_fewer_than_three_warmup_steps_are_refused():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "2")
    assert r.returncode != 0 and "warmup" in r.stderr


def test_roofline_arithmetic_matches_the_stated_figures():
    """Algorithmic bytes and useful flops of the long-context forward, as
    stated for the roofline: 3080 B per token (bf16 q/k/v/h, fp32 otilde per
    element, two fp32 gates) plus the final fp32 state, 405.8 MB per forward;
    B*NH*S*(4 DH^2 + 2 (L+1) DH) useful flops, 3.87e10 at L = 64."""
    sys.path.insert(0, ROOT)
    import bench
    from linear_rnn_mlstm_b200 import synthetic as syn
    w = syn.LONG
    assert bench.fwd_token_bytes(w.DH, 2) == 3080
    per_step = w.B * w.NH * w.S * bench.fwd_token_bytes(w.DH, 2) + bench.state_bytes(w.B * w.NH, w.DH)
    assert abs(per_step / 1e6 - 405.8) < 0.05
    assert bench.kernel_algorithmic_bytes("segment_output_tc", w, {"P": 9}) == per_step
    assert bench.kernel_algorithmic_bytes("gate_prologue", w, {"P": 9}) == w.B * w.NH * w.S * 12
    flops = bench.fwd_flops(w.B * w.NH, w.S, w.DH, 64)
    assert abs(flops / 1e10 - 3.87) < 0.005
