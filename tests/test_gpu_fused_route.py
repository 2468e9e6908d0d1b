"""Gating with the routing counts taken in its epilogue
(tk_gating_fused_topk_route), on the GPU.

* scores and ids are bit-identical to tk_gating_fused_topk's (the same kernels;
  the counting only adds atomic adds after the stores), and on the small shapes
  they also pass the parity rule against the gating oracle directly;
* offsets, sorted_slots and slot_pos are bit-exact against the routing oracle
  (a stable counting sort) applied to the GPU's ids;
* the workspace holds zeros again after every call, so repeated calls and CUDA
  graph replays give the same results;
* stale counts in the workspace are reported (bit 6 of the device error word),
  nothing is written outside the outputs, and the table is zero again; a
  workspace never zeroed at all is reported the same way.

Shapes cover every gating kernel (one-CTA row tiles, CTA pairs with a half-tile
tail, split-H clusters, two expert groups) and both routing plans (one CTA
without a table, several CTAs reading the gating's table), with ragged last
ranges.
"""
import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu

SENTINEL = -7
GUARD = 64
ERR_ROUTE_COUNTS = 1 << 6


@pytest.fixture(scope="module", autouse=True)
def clean_error_word():
    assert torch.cuda.is_available()
    tk.device_error(clear=True)
    yield
    assert tk.device_error(clear=True) == 0


def _guarded(n, fill=SENTINEL):
    return torch.full((n + GUARD,), fill, dtype=torch.int32, device="cuda")


class Fused:
    """Inputs on the device, guarded outputs and a workspace, and the call."""

    def __init__(self, wl: workloads.RouterWorkload):
        self.wl = wl
        self.x = workloads.to_torch_bf16(wl.hidden()).cuda()
        self.w = workloads.to_torch_bf16(wl.gate_weight()).cuda()
        T, k, E = wl.T, wl.k, wl.E
        self.n = T * k
        self.scores = torch.empty(T * k + GUARD, dtype=torch.float32, device="cuda")
        self.ids = _guarded(self.n)
        self.off, self.ss, self.sp = _guarded(E + 1), _guarded(self.n), _guarded(self.n)
        self.plan = tk.route_plan(T, k, E, torch.cuda.get_device_properties(0).multi_processor_count)
        self.ws = tk.route_workspace(T, k, E)
        assert self.ws.numel() * 4 >= self.plan["fused_workspace_bytes"]

    def call(self, stream=0):
        wl = self.wl
        st = tk.fused_topk_gating_route_ptr(
            self.x.data_ptr(), self.w.data_ptr(), wl.T, wl.H, wl.E, wl.k, self.scores.data_ptr(),
            self.ids.data_ptr(), self.off.data_ptr(), self.ss.data_ptr(), self.sp.data_ptr(), self.ws.data_ptr(),
            self.ws.numel() * 4, stream)
        assert st == tk.TK_OK, tk.status_string(st)

    def results(self):
        torch.cuda.synchronize()
        n, E = self.n, self.wl.E
        ids, off, ss, sp = (t.cpu().numpy() for t in (self.ids, self.off, self.ss, self.sp))
        for name, a, m in (("ids", ids, n), ("offsets", off, E + 1), ("sorted_slots", ss, n), ("slot_pos", sp, n)):
            assert (a[m:] == SENTINEL).all(), f"{name}: wrote past its end"
        scores = self.scores.cpu().numpy()[:n].reshape(self.wl.T, self.wl.k)
        return scores, ids[:n].reshape(self.wl.T, self.wl.k), off[:E + 1], ss[:n], sp[:n]

    def workspace_is_zero(self):
        torch.cuda.synchronize()
        return int(torch.count_nonzero(self.ws).item()) == 0


def check_routing(ids, off, ss, sp, E):
    ref = oracle.route(ids, E)
    placed = int(ref.offsets[E])
    assert np.array_equal(off, ref.offsets), "offsets differ"
    assert np.array_equal(sp, ref.slot_pos.reshape(-1)), "slot_pos differs"
    assert np.array_equal(ss[:placed], ref.sorted_slots[:placed]), "sorted_slots differ"


SHAPES = [
    # (T, H, E, k, kind): kernel / routing plan
    (64, 512, 16, 2, "normal"),        # split-H, one routing CTA (no table)
    (1, 7168, 256, 8, "normal"),       # decode, one routing CTA
    (600, 7168, 256, 8, "normal"),     # split-H, two routing CTAs, the second ragged
    (4096, 7168, 256, 8, "normal"),    # the DeepSeek router shape: split-H, 8 routing CTAs
    (16384, 4096, 64, 6, "skew"),      # one-CTA row tiles, ties and duplicated columns
    (65536, 7168, 256, 8, "normal"),   # CTA pairs with 68 half tiles, 128 routing CTAs
    (65533, 2048, 256, 8, "normal"),   # ragged last tile and range
    (3001, 1024, 1024, 16, "normal"),  # two expert groups, k = 16
]


def _wl(T, H, E, k, kind):
    if kind == "skew":
        return workloads.SKEW.with_T(T)
    return workloads.RouterWorkload(f"fused_route_{T}x{H}x{E}x{k}", T, H, E, k, seed=T + E)


@pytest.mark.parametrize("T,H,E,k,kind", SHAPES)
def test_fused_route_matches_separate_calls(T, H, E, k, kind):
    f = Fused(_wl(T, H, E, k, kind))
    assert (f.plan["ctas"] > 1) == (T * k > 4096)
    for _ in range(2):  # the second call runs on the workspace the first one left
        f.call()
        scores, ids, off, ss, sp = f.results()
        assert f.workspace_is_zero(), "the call left counts in the workspace"
        # the separate calls on the same inputs
        s2, i2 = tk.fused_topk_gating(f.x, f.w, k)
        torch.cuda.synchronize()
        assert np.array_equal(ids, i2.cpu().numpy()), "ids differ from tk_gating_fused_topk's"
        assert np.array_equal(scores.view(np.uint32), s2.cpu().numpy().view(np.uint32)), "scores differ"
        check_routing(ids, off, ss, sp, E)
    assert tk.device_error(clear=True) == 0


@pytest.mark.parametrize("T,H,E,k,kind", [s for s in SHAPES if s[0] * s[1] <= 4096 * 7168 and s[4] == "normal"])
def test_fused_route_gating_against_oracle(T, H, E, k, kind):
    wl = _wl(T, H, E, k, kind)
    f = Fused(wl)
    f.call()
    scores, ids, off, ss, sp = f.results()
    ref = oracle.fused_topk_gating(wl.hidden(), wl.gate_weight(), k, want_logits=True)
    parity.check(scores, ids, ref, label=f"fused route {T}x{H}x{E}x{k}")
    check_routing(ids, off, ss, sp, E)


def test_fused_route_in_a_cuda_graph():
    f = Fused(_wl(4096, 7168, 256, 8, "normal"))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        f.call(s.cuda_stream)  # warm-up outside the capture (per-device set-up)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        f.call(s.cuda_stream)
    for v in (f.off, f.ss, f.sp):
        v[:] = SENTINEL
    for _ in range(3):
        g.replay()
    scores, ids, off, ss, sp = f.results()
    assert f.workspace_is_zero()
    check_routing(ids, off, ss, sp, 256)
    del g


def _junk(n, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randint(-1000, 1000, (n,), generator=g, dtype=torch.int32).cuda()


def test_stale_counts_are_reported_and_cleared():
    # A counts table holding stale counts (its arrival counter zero): the
    # placing kernel's check of its table row against its own count of the ids
    # sets bit 6; positions computed from the stale table are only written
    # inside [0, T*k); the last CTA still zeroes the table, so the next call is
    # correct.
    f = Fused(_wl(4096, 7168, 256, 8, "normal"))
    table_words = f.plan["workspace_bytes"] // 4
    f.ws[:table_words] = _junk(table_words, 5)
    f.call()
    torch.cuda.synchronize()
    assert tk.device_error(clear=True) & ERR_ROUTE_COUNTS
    f.results()  # no write past any output's end
    assert f.workspace_is_zero()
    f.call()
    scores, ids, off, ss, sp = f.results()
    assert tk.device_error(clear=True) == 0
    check_routing(ids, off, ss, sp, 256)


def test_workspace_never_zeroed_is_reported():
    # A workspace that was never zeroed, arrival counter included: reported, and
    # nothing written outside the outputs; zeroing it makes the next call correct.
    f = Fused(_wl(4096, 7168, 256, 8, "normal"))
    f.ws.copy_(_junk(f.ws.numel(), 6))
    f.call()
    torch.cuda.synchronize()
    assert tk.device_error(clear=True) & ERR_ROUTE_COUNTS
    f.results()
    f.ws.zero_()
    f.call()
    scores, ids, off, ss, sp = f.results()
    assert tk.device_error(clear=True) == 0
    assert f.workspace_is_zero()
    check_routing(ids, off, ss, sp, 256)


def test_binding_keeps_a_workspace_per_stream():
    wl = _wl(600, 7168, 256, 8, "normal")
    x = workloads.to_torch_bf16(wl.hidden()).cuda()
    w = workloads.to_torch_bf16(wl.gate_weight()).cuda()
    a = tk.fused_topk_gating_route(x, w, 8)
    b = tk.fused_topk_gating_route(x, w, 8)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    check_routing(a[1].cpu().numpy(), a[2].cpu().numpy(), a[3].cpu().numpy(), a[4].cpu().numpy().reshape(-1), 256)


def test_rejects_small_or_missing_workspace():
    f = Fused(_wl(600, 7168, 256, 8, "normal"))
    wl = f.wl
    need = f.plan["fused_workspace_bytes"]
    assert need > 0
    for ws, nbytes in ((0, need), (f.ws.data_ptr(), need - 4)):
        st = tk.fused_topk_gating_route_ptr(
            f.x.data_ptr(), f.w.data_ptr(), wl.T, wl.H, wl.E, wl.k, f.scores.data_ptr(), f.ids.data_ptr(),
            f.off.data_ptr(), f.ss.data_ptr(), f.sp.data_ptr(), ws, nbytes, 0)
        assert st == tk.TK_ERR_INVALID_ARG
    st = tk.fused_topk_gating_route_ptr(
        f.x.data_ptr(), f.w.data_ptr(), wl.T, wl.H, wl.E, wl.k, f.scores.data_ptr(), f.ids.data_ptr(),
        f.off.data_ptr(), f.ss.data_ptr(), f.sp.data_ptr(), f.ws.data_ptr() + 4, need, 0)
    assert st == tk.TK_ERR_ALIGNMENT
    torch.cuda.synchronize()
    assert (f.ids.cpu().numpy() == SENTINEL).all(), "a rejected call wrote"
