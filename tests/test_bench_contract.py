"""bench.py's JSON line carries the keys its consumers read: the reference arm
(the CPU oracle) on CPU, and the GPU arm on a GPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=900):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=timeout, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) >= 1, out.stdout[-2000:]
    return [json.loads(l) for l in lines]


def _common(d):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["config"]["workload"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1 and cb["sample"]
    for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert k in d["e2e"], k


def test_reference_arm_line():
    (d,) = _run("--impl", "reference", "--steps", "2", "--warmup", "1", "--ref-rows", "16")
    _common(d)
    assert d["impl"] == "reference"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["value"] == d["value"]


@pytest.mark.gpu
def test_gpu_arm_line():
    (d,) = _run("--steps", "3", "--warmup", "3", "--cpu-rows", "64")
    _common(d)
    assert "impl" not in d
    rf = d["roofline"]
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s" and 0.3 < rf["frac"] < 1.3
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-3
    assert d["gpu_launches"] == 3                       # one fused launch per timed step
    # per-step spread beside the mean
    assert 0 < d["ms_per_step_min"] <= d["ms_per_step_median"]
    assert d["ms_per_step_min"] <= d["ms_per_step"] * 1.001
    # the staged pipeline's roofline on the same inputs, in the same line
    st = rf["staged"]
    assert st["algorithmic_bytes_per_step"] == 1368391680     # the 70B-shaped INT8 workload, staged
    assert 0.3 < st["frac"] < 1.3 and abs(st["frac"] - st["achieved"] / rf["peak"]) < 1e-3
    assert abs(st["us_per_allreduce"] - sum(st["kernels_us"].values())) < 0.05
    assert st["gpu_launches"] == 3 * (4 + 2)
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])
    assert d["quality"]["bit_exact_vs_oracle"] is True
