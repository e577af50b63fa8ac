"""The JSON line of bench.py, as the benchmark driver reads it: one line per
run with the metric, the throughput, the timing settings, the roofline and
CPU-baseline objects, the end-to-end figure and the clocks.  The reference
arm (the oracle on the host cores) runs without a GPU; the GPU arm needs one.
"""
import json
import os
import subprocess
import sys

import pytest

from conftest import ROOT


def _run(args, timeout):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def _common(line, steps, warmup):
    assert isinstance(line["metric"], str) and line["metric"]
    assert line["value"] > 0 and isinstance(line["unit"], str)
    assert line["n_gpus"] == 1 and line["steps"] == steps and line["warmup"] == warmup
    assert line["ms_per_step"] > 0
    assert line["higher_is_better"] is True
    assert line["scaling"] == "weak"
    assert line["vs_baseline"] is None  # the pages print no figure for this metric
    assert line["data"] == "synthetic"
    cfg = line["config"]
    assert isinstance(cfg["workload"], str) and "l2" in cfg


def test_reference_arm_line_on_the_host():
    line = _run(["--impl", "reference", "--steps", "3", "--warmup", "3", "--workload", "tiny"],
                timeout=600)
    _common(line, 3, 3)
    assert line["impl"] == "reference"
    assert line["dtype"] == "f64"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


@pytest.mark.gpu
def test_gpu_arm_line():
    line = _run(["--workload", "partial_tail", "--steps", "3", "--warmup", "3", "--no-dense",
                 "--mass-rows", "0", "--no-reuse", "--no-cpu-baseline", "--no-per-workload"],
                timeout=1200)
    _common(line, 3, 3)
    assert line["dtype"] == "bf16"
    rf = line["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s"
    assert rf["peak"] > 0 and 0 < rf["frac"] < 1.5
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-9
    e2e = line["e2e"]
    assert e2e["value"] > 0 and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert e2e["value"] < line["value"]  # the copies are inside its timed region
    assert line["gpu_launches"] > 0
    clk = line["clocks"]
    assert clk["sm_max_mhz"] > 0 and isinstance(clk["reasons"], list)
    fe = line["front_end"]
    assert fe["pool"]["frac_of_hbm"] > 0 and fe["pool_score"]["frac_of_hbm"] > 0
