"""The checked build (libtk_gating_debug.so: the same kernels compiled with
TK_GATING_DEBUG, every guarded index checked, a failed check recorded in the
device error word and its access skipped -- the stand-in for a memory
checker).  A child process loads it (TK_GATING_DEBUG=1), runs every kernel
family, routing and expert-parallel dispatch/combine, and reports the error
word; its results must equal the release library's bit for bit."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
from moe_router_gating_b200 import build as tkbuild

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (T, H, E, k): one CTA per tile, CTA pairs with half tiles, two MMA chunks, two
# expert groups, split-H clusters of 16 / 4 / 8; FP8, the workspace entry
# point's split last round and its few-token kernel below
CASES = [(20000, 512, 64, 4), (20000, 512, 256, 8), (24000, 256, 512, 8), (20000, 256, 1024, 8),
         (1, 7168, 256, 8), (4096, 1024, 256, 8), (300, 520, 40, 3), (300, 256, 1024, 32)]

CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import moe_router_gating_b200 as tk, workloads
from moe_router_gating_b200 import ep
assert tk.library_path().endswith("libtk_gating_debug.so")
out = {}
tk.device_error(clear=True)
for (T, H, E, k) in %r:
    wl = workloads.RouterWorkload("chk", T, H, E, k, seed=31)
    x = workloads.to_torch_bf16(wl.hidden()).cuda(); w = workloads.to_torch_bf16(wl.gate_weight()).cuda()
    s, i = tk.fused_topk_gating(x, w, k)
    off, ss, sp = tk.route(i, E)
    out[(T, H, E, k)] = [a.cpu().numpy() for a in (s, i, off, ss, sp)]
xq, xs, wq, ws = workloads.fp8_inputs(workloads.RouterWorkload("chk8", 20000, 512, 256, 8, seed=32))
s8, i8 = tk.fused_topk_gating_fp8(*[torch.from_numpy(a).cuda() for a in (xq, xs, wq, ws)], 8)
out["fp8"] = [s8.cpu().numpy(), i8.cpu().numpy()]
wl = workloads.RouterWorkload("chkws", 20000, 7168, 256, 8, seed=33)
x = workloads.to_torch_bf16(wl.hidden()).cuda(); w = workloads.to_torch_bf16(wl.gate_weight()).cuda()
sw, iw = tk.fused_topk_gating(x, w, 8, workspace=tk.gating_workspace(20000, 7168, 256, 8))
out["split"] = [sw.cpu().numpy(), iw.cpu().numpy()]
wl = workloads.RouterWorkload("chkfew", 3, 7168, 200, 8, seed=34)
x = workloads.to_torch_bf16(wl.hidden()).cuda(); w = workloads.to_torch_bf16(wl.gate_weight()).cuda()
sf, i_f = tk.fused_topk_gating(x, w, 8, workspace=tk.gating_workspace(3, 7168, 200, 8))
out["few"] = [sf.cpu().numpy(), i_f.cpu().numpy()]
g = ep.ExpertParallelGroup(64, 512, capacity=20000 * 4)
xt = workloads.to_torch_bf16(workloads.normal_bf16(5, 1, 0, 20000 * 512).reshape(20000, 512)).cuda()
ids = torch.from_numpy(workloads.expert_ids(20000, 4, 64, seed=5, kind="skew")).cuda()
recv, h = g.fused_dispatch(xt, ids)
g.output[:h.recv_rows].copy_(recv)
comb = g.fused_combine(h, torch.full((20000, 4), 0.25, device="cuda"))
out["ep"] = [recv.view(torch.int16).cpu().numpy(), comb.view(torch.int16).cpu().numpy()]
torch.cuda.synchronize()
out["error_word"] = tk.device_error(clear=True)
np.save(sys.argv[2], out, allow_pickle=True)
"""


def test_checked_build_runs_clean_and_matches_release(tmp_path):
    tkbuild.build(debug=True)  # no-op when up to date
    dst = str(tmp_path / "checked.npy")
    env = dict(os.environ, TK_GATING_DEBUG="1")
    subprocess.run([sys.executable, "-c", CHILD % (CASES,), ROOT, dst], env=env, check=True, timeout=900)
    got = np.load(dst, allow_pickle=True).item()
    assert got["error_word"] == 0, f"checked build reported {got['error_word']:#x}"
    import workloads
    from moe_router_gating_b200 import ep
    for (T, H, E, k) in CASES:
        wl = workloads.RouterWorkload("chk", T, H, E, k, seed=31)
        x = workloads.to_torch_bf16(wl.hidden()).cuda()
        w = workloads.to_torch_bf16(wl.gate_weight()).cuda()
        s, i = tk.fused_topk_gating(x, w, k)
        off, ss, sp = tk.route(i, E)
        for a, b in zip((s, i, off, ss, sp), got[(T, H, E, k)]):
            assert np.array_equal(a.cpu().numpy(), b), (T, H, E, k)
    xq, xs, wq, ws = workloads.fp8_inputs(workloads.RouterWorkload("chk8", 20000, 512, 256, 8, seed=32))
    s8, i8 = tk.fused_topk_gating_fp8(*[torch.from_numpy(a).cuda() for a in (xq, xs, wq, ws)], 8)
    assert np.array_equal(s8.cpu().numpy(), got["fp8"][0]) and np.array_equal(i8.cpu().numpy(), got["fp8"][1])
    # the split last round of the workspace entry point (its own kernel instance)
    wl = workloads.RouterWorkload("chkws", 20000, 7168, 256, 8, seed=33)
    x = workloads.to_torch_bf16(wl.hidden()).cuda()
    w = workloads.to_torch_bf16(wl.gate_weight()).cuda()
    sw, iw = tk.fused_topk_gating(x, w, 8, workspace=tk.gating_workspace(20000, 7168, 256, 8))
    assert np.array_equal(sw.cpu().numpy(), got["split"][0]) and np.array_equal(iw.cpu().numpy(), got["split"][1])
    # the few-token kernel of the workspace entry point (3 tokens, E not a multiple of 32)
    wl = workloads.RouterWorkload("chkfew", 3, 7168, 200, 8, seed=34)
    x = workloads.to_torch_bf16(wl.hidden()).cuda()
    w = workloads.to_torch_bf16(wl.gate_weight()).cuda()
    sf, i_f = tk.fused_topk_gating(x, w, 8, workspace=tk.gating_workspace(3, 7168, 200, 8))
    assert np.array_equal(sf.cpu().numpy(), got["few"][0]) and np.array_equal(i_f.cpu().numpy(), got["few"][1])
    g = ep.ExpertParallelGroup(64, 512, capacity=20000 * 4)
    xt = workloads.to_torch_bf16(workloads.normal_bf16(5, 1, 0, 20000 * 512).reshape(20000, 512)).cuda()
    ids = torch.from_numpy(workloads.expert_ids(20000, 4, 64, seed=5, kind="skew")).cuda()
    recv, h = g.fused_dispatch(xt, ids)
    g.output[:h.recv_rows].copy_(recv)
    comb = g.fused_combine(h, torch.full((20000, 4), 0.25, device="cuda"))
    assert np.array_equal(recv.view(torch.int16).cpu().numpy(), got["ep"][0])
    assert np.array_equal(comb.view(torch.int16).cpu().numpy(), got["ep"][1])
    assert tk.device_error(clear=True) == 0
