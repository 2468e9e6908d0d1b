"""Host-side tooling: the launch-list summary of an ncu CSV, and the digest that
ties a profiled traffic figure to the gating kernels' code (comments ignored)."""
import os

import moe_router_gating_b200.build as tkbuild
from moe_router_gating_b200 import ncu_summary


def test_launch_list_shares(tmp_path):
    csv = tmp_path / "launches.csv"
    csv.write_text(
        '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'
        '"0","void k_a<8>(P)","gpu__time_duration.sum","usecond","30"\n'
        '"1","void k_b(P)","gpu__time_duration.sum","nsecond","10,000"\n'
        '"2","void k_a<8>(P)","gpu__time_duration.sum","usecond","30"\n')
    text = ncu_summary.launches(str(csv))
    lines = text.splitlines()[2:]
    assert lines[0].startswith("void k_a<8> | 2 |")
    assert lines[0].endswith("| 85.7%")
    assert lines[1].startswith("void k_b | 1 |")


def test_digest_ignores_comments_only(tmp_path, monkeypatch):
    for name in tkbuild.GATING_KERNEL_SOURCES:
        (tmp_path / name).write_text(open(os.path.join(tkbuild.CSRC, name)).read())
    monkeypatch.setattr(tkbuild, "CSRC", str(tmp_path))
    d0 = tkbuild.gating_kernel_digest()
    f = tmp_path / "gating_row_tiles.cuh"
    f.write_text("// a new comment line\n" + f.read_text().replace("namespace tkg {", "namespace tkg {  /* note */"))
    assert tkbuild.gating_kernel_digest() == d0
    f.write_text(f.read_text().replace("constexpr int BLOCK_K = 64;", "constexpr int BLOCK_K = 65;"))
    assert tkbuild.gating_kernel_digest() != d0
