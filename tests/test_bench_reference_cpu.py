"""bench.py's reference arm (the fp64 oracle on the host cores) prints one JSON
line with the contract's keys, for the forward and the backward pass."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


@pytest.mark.parametrize("extra", [[], ["--pass", "bwd"], ["--dropout", "0.1"]], ids=["fwd", "bwd", "dropout"])
def test_reference_arm_json_line(extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "c1", "--steps", "2",
           "--warmup", "3", "--cpu-seconds", "0.2"] + extra
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert KEYS <= set(line)
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["higher_is_better"] is True and line["steps"] == 2 and line["warmup"] == 3
    assert "workload" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    if "bwd" in extra:
        assert line["metric"].startswith("attention bwd")
    if "--dropout" in extra:
        assert "dropout" in line["config"]["workload"]
