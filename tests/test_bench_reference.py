"""The reference arm of bench.py (the float64 oracle on the host cores) and the JSON line
it prints: the fields the measurement contract asks of it (CPU only, a few seconds of
oracle time)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--reference-seconds", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, out.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference"
    assert rec["metric"].startswith("effective attended TFLOP/s")
    assert rec["unit"] == "TFLOP/s" and rec["higher_is_better"] is True
    assert rec["value"] > 0 and rec["steps"] == 1 and rec["warmup"] == 3 and rec["ms_per_step"] > 0
    assert rec["dtype"] == "f64" and rec["vs_baseline"] is None
    assert "LVSA" in rec["config"]["workload"]
    cb = rec["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == rec["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = rec["e2e"]
    assert e2e["value"] == rec["value"] and e2e["unit"] == rec["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
