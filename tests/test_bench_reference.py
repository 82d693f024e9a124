"""bench.py's reference arm (the fp64 oracle on the host cores) on the CPU: the sizing of
each step's sample from a calibration, and the JSON line the arm prints."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_oracle(fixed, per_row, max_rows, calls):
    def run(rows):
        calls.append(rows)
        return {"seconds": fixed + per_row * rows, "flops": 10.0 * rows, "sample": f"{rows} rows"}

    run.max_rows = max_rows
    return run


def test_reference_steps_fit_the_budget():
    calls = []
    run = _fake_oracle(0.01, 0.001, 2048, calls)
    secs, flops, rows, sample = bench.reference_steps(run, steps=100, warmup=20)
    per_step = bench.REFERENCE_BUDGET_S / 120
    assert rows == int((per_step - 0.01) / 0.001)  # the fixed per-call cost is not taken per row
    assert calls[4:] == [rows] * 120  # 4 calibration calls, then the warm-up and the timed steps
    assert abs(secs - 100 * (0.01 + 0.001 * rows)) < 1e-9 and flops == 100 * 10.0 * rows
    assert sample == f"{rows} rows"


def test_reference_steps_clamp_the_sample():
    calls = []
    # a call that costs more than a step's share of the budget still runs one row
    assert bench.reference_steps(_fake_oracle(10.0, 0.001, 2048, calls), steps=1000, warmup=20)[2] == 1
    # a cheap oracle with few steps takes the whole workload, no more
    assert bench.reference_steps(_fake_oracle(0.0, 1e-6, 300, calls), steps=3, warmup=3)[2] == 300


def test_reference_arm_json_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--reference-budget", "8"], capture_output=True, text=True, timeout=900,
                         cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1 and line["higher_is_better"]
    assert line["value"] > 0 and line["config"] == bench.config_dict()
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["decode"]["value"] > 0
