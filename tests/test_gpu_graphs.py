"""Gating and routing captured in a CUDA graph and replayed: each replay on new
inputs (copied into the captured buffers) gives exactly the eager result.
Both operators are deterministic (fixed summation order, stable placement),
so the comparison is bit-exact."""
import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,H,E,k", [(4096, 1024, 256, 8), (20000, 512, 256, 8), (3, 2048, 64, 4)])
def test_graph_replay_matches_eager(T, H, E, k):
    dev = torch.device("cuda")
    w = workloads.to_torch_bf16(workloads.RouterWorkload("g", T, H, E, k, seed=1).gate_weight()).to(dev)
    x = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    scores = torch.empty((T, k), dtype=torch.float32, device=dev)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_slots = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot_pos = torch.empty((T, k), dtype=torch.int32, device=dev)

    s = torch.cuda.Stream()
    x.copy_(workloads.to_torch_bf16(workloads.RouterWorkload("g", T, H, E, k, seed=2).hidden()))
    with torch.cuda.stream(s):  # warm-up (first calls set up each device) outside the capture
        tk.fused_topk_gating(x, w, k, scores=scores, ids=ids, stream=s)
        tk.route(ids, E, offsets, sorted_slots, slot_pos, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        tk.fused_topk_gating(x, w, k, scores=scores, ids=ids, stream=s)
        tk.route(ids, E, offsets, sorted_slots, slot_pos, stream=s)

    for seed in (3, 4, 5):
        x.copy_(workloads.to_torch_bf16(workloads.RouterWorkload("g", T, H, E, k, seed=seed).hidden()))
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (scores, ids, offsets, sorted_slots, slot_pos)]
        es, ei = tk.fused_topk_gating(x, w, k)
        eo, ess, esp = tk.route(ei, E)
        torch.cuda.synchronize()
        for a, b in zip(got, (es, ei, eo, ess, esp)):
            assert torch.equal(a, b)
    del g
    assert tk.device_error(clear=True) == 0


@pytest.mark.parametrize("T,H,E,k", [(1, 7168, 256, 8), (4, 2048, 64, 4), (20000, 7168, 256, 8)])
def test_graph_replay_of_workspace_entry_point(T, H, E, k):
    """The workspace entry point captured with its workspace (the few-token kernel's
    arrival counter, the split last round's flags): every replay leaves them zero,
    so replays on new inputs equal eager calls bit for bit."""
    dev = torch.device("cuda")
    w = workloads.to_torch_bf16(workloads.RouterWorkload("gw", T, H, E, k, seed=1).gate_weight()).to(dev)
    x = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    scores = torch.empty((T, k), dtype=torch.float32, device=dev)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    ws = tk.gating_workspace(T, H, E, k)
    assert tk.make_plan_ws(T, H, E, k)[1] > 0  # a plan that uses the workspace

    s = torch.cuda.Stream()
    x.copy_(workloads.to_torch_bf16(workloads.RouterWorkload("gw", T, H, E, k, seed=2).hidden()))
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        tk.fused_topk_gating(x, w, k, scores=scores, ids=ids, stream=s, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        tk.fused_topk_gating(x, w, k, scores=scores, ids=ids, stream=s, workspace=ws)

    for seed in (3, 4):
        x.copy_(workloads.to_torch_bf16(workloads.RouterWorkload("gw", T, H, E, k, seed=seed).hidden()))
        g.replay()
        torch.cuda.synchronize()
        got = (scores.clone(), ids.clone())
        assert not ws[:256].any()
        es, ei = tk.fused_topk_gating(x, w, k, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(got[0], es) and torch.equal(got[1], ei)
    del g
    assert tk.device_error(clear=True) == 0
