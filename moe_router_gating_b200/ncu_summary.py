"""Summarise Nsight Compute output for the profile notes kept under profiles/.

    python -m moe_router_gating_b200.ncu_summary launches <launches.csv> <out.txt> "<command>"
    python -m moe_router_gating_b200.ncu_summary report <raw.csv> <out.txt> "<command>" [--traffic <traffic.txt>]

`launches` turns a `--metrics gpu__time_duration.sum --csv` launch list into per-kernel
launches, total time and share.  `report` picks the figures this project reads from
`ncu -i <rep> --page raw --csv` (DRAM bytes and throughput, tensor-pipe activity, L2,
SM-side stalls, registers); with --traffic it also writes the DRAM bytes per launch
and the digest of the kernel sources, which bench.py reports as the roofline's
`traffic` only while the sources are unchanged.
"""
from __future__ import annotations

import csv
import os
import sys
from collections import OrderedDict

PKG = os.path.dirname(os.path.abspath(__file__))

REPORT_METRICS = [
    "gpu__time_duration.sum",
    "sm__cycles_elapsed.avg.per_second",
    "dram__bytes_read.sum",
    "dram__bytes_write.sum",
    "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed",
    "sm__cycles_active.avg",
    "l1tex__m_xbar2l1tex_read_bytes.sum",
    "lts__t_sector_hit_rate.pct",
    "lts__throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__throughput.avg.pct_of_peak_sustained_elapsed",
    "launch__registers_per_thread",
    "launch__grid_size",
    "launch__cluster_size",
    "smsp__average_warps_issue_stalled_long_scoreboard_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_wait_per_issue_active.ratio",
]


def kernel_source_digest() -> str:
    """Same digest as bench.py: the gating kernels' code, comments ignored."""
    from moe_router_gating_b200 import build as tkbuild
    return tkbuild.gating_kernel_digest()


def _rows(path):
    with open(path, newline="") as f:
        lines = [ln for ln in f if ln.startswith('"')]
    return list(csv.reader(lines))


def launches(csv_path: str) -> str:
    rows = _rows(csv_path)
    hdr = rows[0]
    ki, mi, vi = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    ui = hdr.index("Metric Unit")
    per = OrderedDict()
    for r in rows[1:]:
        if r[mi] != "gpu__time_duration.sum":
            continue
        v = float(r[vi].replace(",", ""))
        unit = r[ui]
        scale_us = {"ns": 1e-3, "nsecond": 1e-3, "us": 1.0, "usecond": 1.0, "ms": 1e3, "msecond": 1e3,
                    "s": 1e6, "second": 1e6}
        if unit not in scale_us:
            raise ValueError(f"unknown time unit {unit!r} in {csv_path}")
        us = v * scale_us[unit]
        name = r[ki].split("(")[0].strip()
        n, t = per.get(name, (0, 0.0))
        per[name] = (n + 1, t + us)
    total = sum(t for _, t in per.values()) or 1.0
    out = ["kernel | launches | total us | share", "---|---|---|---"]
    for name, (n, t) in sorted(per.items(), key=lambda kv: -kv[1][1]):
        out.append(f"{name} | {n} | {t:.1f} | {100 * t / total:.1f}%")
    return "\n".join(out)


def report(raw_csv: str):
    rows = _rows(raw_csv)
    hdr, units = rows[0], rows[1]
    found = OrderedDict()
    for vals in rows[2:]:
        kname = vals[hdr.index("Kernel Name")] if "Kernel Name" in hdr else "?"
        for m in REPORT_METRICS:
            if m in hdr:
                i = hdr.index(m)
                found.setdefault(kname, []).append((m, vals[i], units[i]))
    return found


def main(argv):
    mode = argv[1]
    if mode == "launches":
        src, out, cmd = argv[2], argv[3], argv[4]
        body = launches(src)
        with open(out, "w") as f:
            f.write(f"# Launch list (ncu gpu__time_duration.sum, cold-cache and serialised: compare shares)\n")
            f.write(f"# command: {cmd}\n\n{body}\n")
    elif mode == "report":
        src, out, cmd = argv[2], argv[3], argv[4]
        traffic_out = argv[argv.index("--traffic") + 1] if "--traffic" in argv else None
        found = report(src)
        lines = [f"# ncu --set full summary", f"# command: {cmd}", ""]
        dram = None
        for kname, metrics in found.items():
            lines.append(f"kernel: {kname}")
            rb = wb = None
            for m, v, u in metrics:
                lines.append(f"  {m} = {v} {u}")
                if m == "dram__bytes_read.sum":
                    rb = (v, u)
                if m == "dram__bytes_write.sum":
                    wb = (v, u)
            if rb and wb:
                scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
                dram = float(rb[0].replace(",", "")) * scale[rb[1]] + float(wb[0].replace(",", "")) * scale[wb[1]]
                lines.append(f"  dram bytes per launch (read + write) = {dram:.0f}")
            lines.append("")
        with open(out, "w") as f:
            f.write("\n".join(lines))
        if traffic_out and dram is not None:
            with open(traffic_out, "w") as f:
                f.write("# DRAM bytes (read + write) per launch of the fused gating kernel, from one ncu capture\n")
                f.write(f"# command: {cmd}\n")
                f.write(f"kernel_source_digest = {kernel_source_digest()}\n")
                f.write(f"dram_bytes_per_launch = {dram:.0f}\n")
    else:
        raise SystemExit(__doc__)


if __name__ == "__main__":
    main(sys.argv)
