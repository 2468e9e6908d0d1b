"""The workspace entry points (tk_gating_fused_topk_ws and its FP8 twin) on the
GPU, against the oracle on every row.

Where the plan without workspace ends with a round of 128-token half tiles,
these entry points cut each of the last round's 256-token tiles in H between two
CTA pairs: the first stores its fp32 accumulator rows to the workspace and sets
a flag, the second adds them to its own and selects (the logits step of the
naive form, ``hidden_states @ gate_weight``, on the chenxutan.com page
"TileKernels 深度解析", section 4.1, cut along H for those rows).  Checked here:

* the parity rule against the oracle on every row of the train shape, of a
  ragged T whose last split tile is partly past T, of T = 20000, and on FP8;
* the logit error budget and bit-identical logits of duplicated gate columns in
  the split rows;
* the flags are left zero by every call, so repeated calls on one workspace give
  the same results; nothing is written outside scores and ids;
* a missing, small or misaligned workspace is rejected before any launch; where
  nothing is split the call is tk_gating_fused_topk's, bitwise, and the
  workspace may be NULL;
* an expired wait (the flag or the staged rows) is reported and the context
  survives.
"""
import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import oracle
import parity
import workloads
from gpu_helpers import to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def clean_error_word():
    assert torch.cuda.is_available()
    tk.device_error(clear=True)
    yield
    assert tk.device_error(clear=True) == 0, "a kernel wait expired during the GPU tests"


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def split_rows(T, H, E, k):
    """First row of the split tiles and their count (0 when nothing is split)."""
    plan, nbytes = tk.make_plan_ws(T, H, E, k, _sms())
    return plan["num_tiles"] * 256, plan["num_split_tiles"], nbytes


def flag_bytes(n_split):
    """The workspace's leading flags: 8 bytes per split tile, rounded up to 256."""
    return (n_split * 8 + 255) // 256 * 256


def run_ws(x_bits, w_bits, k, logits=False):
    x, w = to_device_bf16(x_bits), to_device_bf16(w_bits)
    T, H = x_bits.shape
    E = w_bits.shape[1]
    ws = tk.gating_workspace(T, H, E, k)
    L = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda") if logits else None
    s, i = tk.fused_topk_gating(x, w, k, workspace=ws, logits=L)
    torch.cuda.synchronize()
    flags = ws[:flag_bytes(split_rows(T, H, E, k)[1])].cpu().numpy()
    assert not flags.any(), "the call left a split flag set"
    return s.cpu().numpy(), i.cpu().numpy(), (L.cpu().numpy() if logits else None)


@pytest.mark.parametrize("T,H,E,k", [
    (65536, 7168, 256, 8),   # the train shape: 34 split tiles
    (20000, 7168, 256, 8),   # one full round, 5 split tiles
    (65533, 6144, 200, 6),   # ragged: the last split tile's second CTA holds rows past T
    (23000, 6144, 136, 1),   # k = 1, E padded inside the pair halves
])
def test_split_last_round_matches_oracle(T, H, E, k):
    first, n_split, nbytes = split_rows(T, H, E, k)
    assert n_split > 0 and nbytes > 0
    wl = workloads.RouterWorkload(f"split_{T}_{H}_{E}_{k}", T, H, E, k, seed=T % 97)
    x_bits, w_bits = wl.hidden(), wl.gate_weight()
    s, i, _ = run_ws(x_bits, w_bits, k)
    ref = oracle.fused_topk_gating(x_bits, w_bits, k, want_logits=True)
    info = parity.check(s, i, ref, label=wl.name)
    assert info["rows"] == T
    assert np.all(np.abs(s.astype(np.float64).sum(axis=1) - 1.0) <= 1e-5)


def test_logit_error_and_duplicate_columns_in_split_rows():
    T, H, E, k = 20000, 7168, 256, 8
    first, n_split, _ = split_rows(T, H, E, k)
    wl = workloads.RouterWorkload("split_dups", T, H, E, k, seed=12)
    w_bits = wl.gate_weight().copy()
    pairs = ((3, 200), (64, 65), (127, 128), (10, 250))  # across the CTA pair's gate halves too
    for a, b in pairs:
        w_bits[:, b] = w_bits[:, a]
    x_bits = wl.hidden()
    s, i, L = run_ws(x_bits, w_bits, k, logits=True)
    assert not np.isnan(L).any()
    for a, b in pairs:
        assert np.array_equal(L[:, a].view(np.uint32), L[:, b].view(np.uint32))
    ref = oracle.fused_topk_gating(x_bits, w_bits, k, want_logits=True)
    err = parity.logit_error(L, ref.logits)
    err_split = parity.logit_error(L[first:], ref.logits[first:])
    print(f"\nsplit last round: max |logit error| {err:.3e} (split rows {err_split:.3e})")
    assert err <= parity.LOGIT_ATOL
    parity.check_own_selection(s, i, L, label="split_dups")
    parity.check(s, i, ref, duplicate_pairs=pairs, label="split_dups")


def test_repeated_calls_and_nothing_outside_the_outputs():
    wl = workloads.RouterWorkload("split_guard", 20000, 7168, 256, 8, seed=2)
    x, w = to_device_bf16(wl.hidden()), to_device_bf16(wl.gate_weight())
    ws = tk.gating_workspace(wl.T, wl.H, wl.E, wl.k)
    pad = 64
    n = wl.T * wl.k
    s_buf = torch.full((n + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    i_buf = torch.full((n + 2 * pad,), -7, dtype=torch.int32, device="cuda")
    s = s_buf[pad:pad + n].view(wl.T, wl.k)
    i = i_buf[pad:pad + n].view(wl.T, wl.k)
    outs = []
    for _ in range(3):
        tk.fused_topk_gating(x, w, wl.k, scores=s, ids=i, workspace=ws)
        outs.append((s.clone(), i.clone()))
    torch.cuda.synchronize()
    assert torch.all(s_buf[:pad] == 7.0) and torch.all(s_buf[-pad:] == 7.0)
    assert torch.all(i_buf[:pad] == -7) and torch.all(i_buf[-pad:] == -7)
    for s1, i1 in outs[1:]:
        assert torch.equal(s1, outs[0][0]) and torch.equal(i1, outs[0][1])
    assert not ws[:flag_bytes(split_rows(wl.T, wl.H, wl.E, wl.k)[1])].any()
    # the rows before the split round are the plain call's, bitwise
    s0, i0 = tk.fused_topk_gating(x, w, wl.k)
    first, _, _ = split_rows(wl.T, wl.H, wl.E, wl.k)
    torch.cuda.synchronize()
    assert torch.equal(s0[:first], outs[0][0][:first]) and torch.equal(i0[:first], outs[0][1][:first])


def test_bad_workspace_is_rejected_before_any_launch():
    T, H, E, k = 20000, 7168, 256, 8
    wl = workloads.RouterWorkload("split_bad", T, H, E, k, seed=1)
    x, w = to_device_bf16(wl.hidden()), to_device_bf16(wl.gate_weight())
    need = tk.workspace_bytes(T, H, E, k)
    assert need == split_rows(T, H, E, k)[2] > 0
    ws = torch.zeros(need + 16, dtype=torch.uint8, device="cuda")
    s = torch.full((T, k), 7.0, dtype=torch.float32, device="cuda")
    i = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    call = lambda p, nb: tk.fused_topk_gating_ws_ptr(x.data_ptr(), w.data_ptr(), T, H, E, k, s.data_ptr(),
                                                     i.data_ptr(), p, nb, 0)
    assert call(0, need) == tk.TK_ERR_INVALID_ARG
    assert call(ws.data_ptr(), need - 16) == tk.TK_ERR_INVALID_ARG
    assert call(ws.data_ptr(), -1) == tk.TK_ERR_INVALID_ARG
    assert call(ws.data_ptr() + 8, need) == tk.TK_ERR_ALIGNMENT
    torch.cuda.synchronize()
    assert torch.all(s == 7.0) and torch.all(i == -7), "a rejected call wrote"
    assert call(ws.data_ptr(), need) == tk.TK_OK
    torch.cuda.synchronize()


@pytest.mark.parametrize("T,H,E,k", [(4096, 7168, 256, 8), (65536, 2048, 256, 8), (65536, 7168, 512, 8),
                                     (60000, 4096, 256, 16), (16384, 4096, 64, 6)])
def test_without_a_split_the_call_is_the_plain_one(T, H, E, k):
    wl = workloads.RouterWorkload(f"nosplit_{T}_{H}_{E}_{k}", T, H, E, k, seed=3)
    x, w = to_device_bf16(wl.hidden()), to_device_bf16(wl.gate_weight())
    assert tk.workspace_bytes(T, H, E, k) == 0
    assert tk.make_plan_ws(T, H, E, k, _sms()) == (tk.make_plan(T, H, E, k, _sms()), 0)
    s0, i0 = tk.fused_topk_gating(x, w, k)
    s = torch.empty_like(s0)
    i = torch.empty_like(i0)
    assert tk.fused_topk_gating_ws_ptr(x.data_ptr(), w.data_ptr(), T, H, E, k, s.data_ptr(), i.data_ptr(),
                                       0, 0, 0) == tk.TK_OK
    torch.cuda.synchronize()
    assert torch.equal(s, s0) and torch.equal(i, i0)


def test_fp8_split_last_round_matches_fp8_oracle():
    # FP8 slices hold 128 values of H: H = 12288 gives the 96 slices the split needs
    T, H, E, k = 20000, 12288, 256, 8
    wl = workloads.RouterWorkload("split_fp8", T, H, E, k, seed=9)
    assert tk.make_plan_ws(T, H // 2, E, k, _sms())[0]["num_split_tiles"] > 0
    xq, xs, wq, wsc = workloads.fp8_inputs(wl)
    dev = [torch.from_numpy(a).cuda() for a in (xq, xs, wq, wsc)]
    work = tk.gating_workspace(T, H, E, k, fp8=True)
    s, i = tk.fused_topk_gating_fp8(*dev, k, workspace=work)
    torch.cuda.synchronize()
    assert not work[:flag_bytes(tk.make_plan_ws(T, H // 2, E, k, _sms())[0]["num_split_tiles"])].any()
    ref = oracle.fused_topk_gating_fp8(xq, xs, wq, wsc, k, want_logits=True)
    parity.check(s.cpu().numpy(), i.cpu().numpy(), ref, label=wl.name)


def test_expired_wait_is_reported_and_context_survives():
    T, H, E, k = 20000, 7168, 256, 8
    wl = workloads.RouterWorkload("split_abort", T, H, E, k, seed=8)
    x_bits, w_bits = wl.hidden(), wl.gate_weight()
    x, w = to_device_bf16(x_bits), to_device_bf16(w_bits)
    ws = tk.gating_workspace(T, H, E, k)
    tk.device_error(clear=True)
    tk.set_wait_timeout_ns(1000)
    try:
        tk.fused_topk_gating(x, w, k, workspace=ws)
        torch.cuda.synchronize()
    finally:
        tk.set_wait_timeout_ns(1_000_000_000)
    assert tk.device_error(clear=True) != 0, "a 1 us wait limit must expire during this launch"
    ws.zero_()  # an aborted call may leave a flag set
    s, i = tk.fused_topk_gating(x, w, k, workspace=ws)
    torch.cuda.synchronize()
    assert tk.device_error(clear=True) == 0
    first, _, _ = split_rows(T, H, E, k)
    rows = np.unique(np.concatenate([np.arange(0, first, 151), np.arange(first, T, 3)]))
    ref = oracle.fused_topk_gating(x_bits[rows], w_bits, k, want_logits=True)
    parity.check(s.cpu().numpy(), i.cpu().numpy(), ref, rows=rows, label="split after-timeout")
