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


def test_roofline_reports_both_tensor_peaks():
    import bench
    import workloads
    peaks = {"hbm_gbs": 6532.5, "bf16_tflops": 1672.3, "bf16_tflops_sustained": 1400.0}
    wl = workloads.TRAIN
    r = bench.roofline_of(wl, 0.2, False, peaks, "test")
    t_hbm = wl.algorithmic_bytes() / 6532.5e9
    t_tc = wl.flops() / 1672.3e12
    t_tcs = wl.flops() / 1400.0e12
    assert r["bound"] == ("hbm" if t_hbm >= t_tc else "tensor")
    assert abs(r["roofline_frac"] - max(t_hbm, t_tc) / 2e-4) < 1e-12
    assert abs(r["roofline_frac_sustained"] - max(t_hbm, t_tcs) / 2e-4) < 1e-12
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    # the FP8 roofline counts 1-byte operands and doubles the tensor peak
    r8 = bench.roofline_of(wl, 0.2, True, peaks, "test")
    assert r8["algorithmic_bytes_per_launch"] < wl.algorithmic_bytes() // 2 + 10 * wl.T * wl.k
    assert abs(r8["roofline_us"]["tensor_burst"] - t_tc * 1e6 / 2) < 1e-6
