"""bench.py's output contract, checked on the CPU through its reference arm.

The reference arm times the CPU oracle and prints the same single JSON line as
the GPU arm, so the keys and types the benchmark driver reads can be checked
without a GPU: one JSON line on stdout, the metric, the unit, the per-step time,
the e2e object and the cpu_baseline description.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = _run("--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3")
    assert d["impl"] == "reference"
    assert d["metric"] == "signsgd_steps_per_sec" and d["unit"] == "steps/s"
    assert d["higher_is_better"] is True and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["data"] == "synthetic" and d["config"]["workload"].startswith("tiny")
    # the same config, key for key, as the GPU arm states for this workload
    sys.path.insert(0, ROOT)
    import bench
    assert d["config"] == json.loads(json.dumps(bench._config(bench.WORKLOADS["tiny"], 1)))
    for key in ("lr", "minmax_lr", "keep_best", "batch_rows", "iters", "bits", "group_size", "sym"):
        assert key in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_rejects_short_warmup():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], cwd=ROOT,
                         capture_output=True, text=True, timeout=120)
    assert out.returncode != 0


def test_gemm_fingerprint_ignores_comments_only():
    """The ncu traffic figures stay valid across comment edits, not code edits."""
    sys.path.insert(0, ROOT)
    import bench
    a = "int f(int x) {  // first\n  /* block */ return x + 1;\n}\n\nconst char* s = \"a//b\";\n"
    b = "// header\nint f(int x) {\n  return x + 1;   // other words\n}\nconst char* s = \"a//b\";\n"
    assert bench._strip_comments(a) == bench._strip_comments(b)
    assert bench._strip_comments(a) != bench._strip_comments(a.replace("x + 1", "x + 2"))
    assert "a//b" in bench._strip_comments(a)
    assert len(bench.gemm_code_fingerprint()) == 16


def test_group_size_override_names_the_workload():
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    c = bench._workload(argparse.Namespace(workload="q_proj", group_size=-1))
    assert c.group_size == -1 and "per-channel" in c.name and "g128" not in c.name
    c = bench._workload(argparse.Namespace(workload="q_proj", group_size=64))
    assert c.group_size == 64 and " g64" in c.name
    c = bench._workload(argparse.Namespace(workload="q_proj", group_size=None))
    assert c is bench.WORKLOADS["q_proj"]


def test_clock_summary_parses_samples():
    """The clocks object: median SM clock and power draw, the max clock, and every throttle
    reason seen active in any sample (nvidia-smi csv, noheader, nounits)."""
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler(0)
    c.lines = ["0, 1500, 1965, 980.5, Not Active, Not Active, Not Active, Active",
               "0, 1440, 1965, 995.0, Not Active, Not Active, Not Active, Active",
               "0, 1470, 1965, 990.0, Not Active, Not Active, Not Active, Not Active",
               "garbage"]
    s = c.summary()
    assert s["sm_mhz"] == 1470 and s["sm_max_mhz"] == 1965 and s["power_w"] == 990.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
