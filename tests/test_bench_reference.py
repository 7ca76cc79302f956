"""The reference arm of bench.py (the oracle on the host cores), CPU only.

Runs `bench.py --impl reference` on the small workloads and checks the JSON
line the benchmark contract asks for: one line, the arm's own metric, unit
and direction, a cpu_baseline describing the run, an e2e entry with no
host-device copies, and a rejected warm-up below 3 steps.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=600, cwd=ROOT)


@pytest.mark.parametrize("workload", ["tiny", "affine"])
def test_reference_arm_json_line(workload):
    r = _run("--impl", "reference", "--workload", workload, "--steps", "3", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["steps"] == 3 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"] == workload
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    rates = cb["rates_by_workload"]          # every workload, one thread and all threads
    assert set(rates) == {"tiny", "gqa", "qjl", "long", "serving", "affine"}
    for r in rates.values():
        for mode in ("all_threads", "one_thread"):
            assert r[mode]["quantize_mvec_s"] > 0 and r[mode]["decode_ctx_tokens_s"] > 0
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_warmup_below_three_is_rejected():
    r = _run("--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "2")
    assert r.returncode != 0 and "warmup" in r.stderr


def test_clock_summary_parses_nvidia_smi_lines():
    """The clocks entry: median SM clock under load, max clock, active reasons."""
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.out = "\n".join([
        "1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "1950, 1965, 900.3, 0x4, Not Active, Not Active, Not Active, Active",
        "1965, 1965, 880.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ])
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    c.out = ""
    assert c.summary()["reasons"] == ["unavailable"]


def test_other_ranks_print_nothing():
    """Under torchrun every rank but 0 exits 0 without work or output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "3", "--warmup", "3", "--gpus", "2"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
