"""The bench's GPU arm keeps the line contract: one JSON line with the driver's keys, the
roofline and end-to-end objects filled, our kernels counted, clocks sampled, no device fault.
Runs the tiny configuration for a few steps (a few seconds)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "roofline",
        "e2e", "clocks", "gpu_launches"}


@pytest.mark.parametrize("extra", [[], ["--kv-fp8", "--workload", "gqa"]])
def test_gpu_arm_prints_one_contract_line(extra):
    args = [sys.executable, "bench.py", "--steps", "4", "--warmup", "3", "--no-cpu-baseline",
            "--no-read-probe"]
    if not extra:
        args += ["--workload", "tiny"]
    out = subprocess.run(args + extra, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, out.stdout[-2000:]
    d = json.loads(lines[0])
    assert KEYS <= set(d), KEYS - set(d)
    assert d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["achieved"] > 0 and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] > 0
    assert isinstance(d["config"], dict) and "workload" in d["config"]
