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


def test_peak_follows_the_sampled_clocks(monkeypatch, tmp_path):
    """The roofline denominator is the burst bf16 figure at full clock and the
    sustained one when the timed region ran power-capped; both kinds are read
    from the peaks file when it has them, else from the fallback figures."""
    sys.path.insert(0, ROOT)
    import bench
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    capped = {"sm_mhz": 1728.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    slow_no_reason = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": []}
    monkeypatch.setattr(bench, "PEAKS_PATH", str(tmp_path / "absent.json"))
    assert bench.peak_tflops(None)[0] == bench.FALLBACK_BF16_TFLOPS
    assert bench.peak_tflops(full)[0] == bench.FALLBACK_BF16_TFLOPS
    assert bench.peak_tflops(slow_no_reason)[0] == bench.FALLBACK_BF16_TFLOPS
    peak, src, burst = bench.peak_tflops(capped)
    assert peak == bench.FALLBACK_BF16_TFLOPS_SUSTAINED and burst == bench.FALLBACK_BF16_TFLOPS
    assert "sustained" in src
    path = tmp_path / "peaks.json"
    path.write_text(json.dumps({"bf16_tflops": 1637.9, "bf16_tflops_sustained": 1420.0, "hbm_gbs": 7000.0}))
    monkeypatch.setattr(bench, "PEAKS_PATH", str(path))
    assert bench.peak_tflops(full)[:1] == (1637.9,)
    assert bench.peak_tflops(capped)[0] == 1420.0 and bench.peak_tflops(capped)[2] == 1637.9


@pytest.mark.parametrize("B,H,n", [(1, 32, 8), (32, 16, 8), (2, 10, 8), (1, 3, 8), (4, 40, 1), (1, 1, 16), (3, 7, 2)])
def test_e2e_chunks_cover_the_axis(B, H, n):
    """The end-to-end step's chunks: whole batches when B > 1, else heads;
    contiguous, in order, covering the axis once, sizes within one."""
    sys.path.insert(0, ROOT)
    import bench
    axis, rng = bench.e2e_chunks(B, H, n)
    total = B if B > 1 else H
    assert axis == ("b" if B > 1 else "h")
    assert len(rng) == max(1, min(n, total))
    pos = 0
    for first, count in rng:
        assert first == pos and count >= 1
        pos += count
    assert pos == total
    sizes = [c for _, c in rng]
    assert max(sizes) - min(sizes) <= 1
