"""The JSON line of bench.py's reference arm (the oracle timed on the host
cores), run on the CPU: every key the launch contract names, with the same
metric, unit and workload as the GPU arm's line."""
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    t0 = time.time()
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, cwd=ROOT, timeout=600)
    wall = time.time() - t0
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])

    sys.path.insert(0, ROOT)
    import bench
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["config"] == bench.CONFIG
    assert line["unit"] == "TFLOPS" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["ms_per_step"] > 0
    # ms_per_step is the sampled step as it ran (it fits in the run's wall
    # time); the metric uses the step extrapolated to all M rows
    assert line["steps"] * line["ms_per_step"] <= wall * 1e3
    assert line["full_step_ms_extrapolated"] >= line["ms_per_step"]
    assert abs(line["value"] - bench.FLOPS / (line["full_step_ms_extrapolated"] * 1e-3) / 1e12) < 1e-9 * line["value"]
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 1, 0)
    assert line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["data"] == "synthetic" and isinstance(line["dtype"], str)
    assert "workload" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["unit"] == line["unit"]
    assert cb["cores"] >= 1 and isinstance(cb["sample"], str) and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
