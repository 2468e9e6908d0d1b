"""The benchmark's reference arm (the CPU oracle, timed on this host) prints the
JSON line the benchmark contract asks for; no GPU is involved."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True, check=True, cwd=ROOT,
                         timeout=300).stdout.strip().splitlines()
    line = json.loads(out[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert "tiny" in line["config"]["workload"]


def test_reference_arm_other_ops_report_unavailable():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--op", "route"],
                         capture_output=True, text=True, check=True, cwd=ROOT, timeout=120).stdout.strip()
    line = json.loads(out.splitlines()[-1])
    assert line["impl"] == "reference" and "unavailable" in line
