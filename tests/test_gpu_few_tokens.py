"""The few-token kernel of the workspace entry point (tk_gating_fused_topk_ws
with 1 <= T <= 4, E <= 256) on the GPU, against the oracle on every row.

About one CTA per SM each accumulates a block of 32 experts over a range of H
on the CUDA cores and stores its partial logits to the workspace; the CTA that
finishes last adds them in the order of the H ranges, selects and stores (the
naive form on the chenxutan.com page "TileKernels 深度解析", section 4.1:
``hidden_states @ gate_weight``, top k, softmax over the k).  Checked here:

* the parity rule against the oracle on every row, over T = 1..4, E from 16 to
  256 (multiples of 8 that are not multiples of 32 too), k from 1 to 32, and H
  whose last range is shorter than the others or a single 8-row range;
* the logit error budget, and bit-identical logits of duplicated gate columns
  (also across the CTAs' expert blocks);
* the counter is zero after every call, so calls of any size may share one
  workspace; repeated calls give bitwise the same outputs; nothing is written
  outside scores and ids;
* the decode workload through the binding that bench.py times.
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

FEW_TOKENS = 4  # plan variant


@pytest.fixture(scope="module", autouse=True)
def clean_error_word():
    assert torch.cuda.is_available()
    tk.device_error(clear=True)
    yield
    assert tk.device_error(clear=True) == 0, "a kernel wait expired during the GPU tests"


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def run_ws(x_bits, w_bits, k, ws=None, logits=False):
    x, w = to_device_bf16(x_bits), to_device_bf16(w_bits)
    T, H = x_bits.shape
    E = w_bits.shape[1]
    plan, nbytes = tk.make_plan_ws(T, H, E, k, _sms())
    assert plan["variant"] == FEW_TOKENS and nbytes > 0
    if ws is None:
        ws = tk.gating_workspace(T, H, E, k)
    L = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda") if logits else None
    s, i = tk.fused_topk_gating(x, w, k, workspace=ws, logits=L)
    torch.cuda.synchronize()
    assert not ws[:256].any(), "the call left its counter non-zero"
    return s.cpu().numpy(), i.cpu().numpy(), (L.cpu().numpy() if logits else None)


@pytest.mark.parametrize("T,H,E,k", [
    (1, 7168, 256, 8),    # the decode workload, one token
    (2, 7168, 256, 8),
    (3, 7168, 256, 8),
    (4, 7168, 256, 8),    # the most tokens this kernel takes
    (3, 4096, 64, 6),     # 74 ranges of 56 rows
    (4, 512, 16, 2),      # half of each expert block past E
    (4, 2048, 200, 8),    # E not a multiple of 32
    (1, 7168, 136, 1),    # k = 1
    (4, 7168, 256, 32),   # lists of 32
    (2, 1000, 96, 16),    # H = 1000: the last range shorter, lists of 16
    (1, 8, 16, 4),        # a single 8-row range
])
def test_few_tokens_match_oracle(T, H, E, k):
    wl = workloads.RouterWorkload(f"few_{T}_{H}_{E}_{k}", T, H, E, k, seed=T * 31 + E)
    x_bits, w_bits = wl.hidden(), wl.gate_weight()
    s, i, L = run_ws(x_bits, w_bits, k, logits=True)
    ref = oracle.fused_topk_gating(x_bits, w_bits, k, want_logits=True)
    info = parity.check(s, i, ref, label=wl.name)
    assert info["rows"] == T
    assert np.all(np.abs(s.astype(np.float64).sum(axis=1) - 1.0) <= 1e-5)
    assert parity.logit_error(L, ref.logits) <= parity.LOGIT_ATOL
    parity.check_own_selection(s, i, L, label=wl.name)


def test_logit_error_and_duplicate_columns():
    T, H, E, k = 4, 7168, 256, 8
    wl = workloads.RouterWorkload("few_dups", T, H, E, k, seed=21)
    w_bits = wl.gate_weight().copy()
    pairs = ((3, 200), (31, 32), (64, 65), (10, 250))  # across the CTAs' 32-expert blocks too
    for a, b in pairs:
        w_bits[:, b] = w_bits[:, a]
    x_bits = wl.hidden()
    s, i, L = run_ws(x_bits, w_bits, k, logits=True)
    assert not np.isnan(L).any()
    for a, b in pairs:
        assert np.array_equal(L[:, a].view(np.uint32), L[:, b].view(np.uint32))
    ref = oracle.fused_topk_gating(x_bits, w_bits, k, want_logits=True)
    err = parity.logit_error(L, ref.logits)
    print(f"\nfew-token kernel: max |logit error| {err:.3e}")
    assert err <= parity.LOGIT_ATOL
    parity.check(s, i, ref, duplicate_pairs=pairs, label="few_dups")


def test_shared_workspace_repeated_calls_and_guard_band():
    # one workspace, large enough for every call below, shared by calls of different sizes in order
    shapes = [(4, 7168, 256, 8), (1, 7168, 256, 8), (3, 4096, 64, 6), (4, 7168, 256, 8)]
    need = max(tk.workspace_bytes(*sh) for sh in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    first = {}
    for n, (T, H, E, k) in enumerate(shapes * 2):
        wl = workloads.RouterWorkload(f"few_share_{T}_{E}", T, H, E, k, seed=4)
        x, w = to_device_bf16(wl.hidden()), to_device_bf16(wl.gate_weight())
        pad = 64
        s_buf = torch.full((T * k + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
        i_buf = torch.full((T * k + 2 * pad,), -7, dtype=torch.int32, device="cuda")
        s = s_buf[pad:pad + T * k].view(T, k)
        i = i_buf[pad:pad + T * k].view(T, k)
        tk.fused_topk_gating(x, w, k, scores=s, ids=i, workspace=ws)
        torch.cuda.synchronize()
        assert not ws[:256].any()
        assert torch.all(s_buf[:pad] == 7.0) and torch.all(s_buf[-pad:] == 7.0)
        assert torch.all(i_buf[:pad] == -7) and torch.all(i_buf[-pad:] == -7)
        key = (T, H, E, k)
        if key in first:  # the same inputs: bitwise the same outputs
            assert torch.equal(s, first[key][0]) and torch.equal(i, first[key][1])
        else:
            first[key] = (s.clone(), i.clone())
            ref = oracle.fused_topk_gating(wl.hidden(), wl.gate_weight(), k, want_logits=True)
            parity.check(s.cpu().numpy(), i.cpu().numpy(), ref, label=wl.name)


def test_small_workspace_is_rejected_and_plain_call_unchanged():
    T, H, E, k = 4, 7168, 256, 8
    wl = workloads.RouterWorkload("few_bad", T, H, E, k, seed=1)
    x, w = to_device_bf16(wl.hidden()), to_device_bf16(wl.gate_weight())
    need = tk.workspace_bytes(T, H, E, k)
    assert need == tk.make_plan_ws(T, H, E, k, _sms())[1] > 0
    ws = torch.zeros(need + 16, dtype=torch.uint8, device="cuda")
    s = torch.full((T, k), 7.0, dtype=torch.float32, device="cuda")
    i = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    call = lambda p, nb: tk.fused_topk_gating_ws_ptr(x.data_ptr(), w.data_ptr(), T, H, E, k, s.data_ptr(),
                                                     i.data_ptr(), p, nb, 0)
    assert call(0, need) == tk.TK_ERR_INVALID_ARG
    assert call(ws.data_ptr(), need - 16) == tk.TK_ERR_INVALID_ARG
    assert call(ws.data_ptr() + 8, need) == tk.TK_ERR_ALIGNMENT
    torch.cuda.synchronize()
    assert torch.all(s == 7.0) and torch.all(i == -7), "a rejected call wrote"
    assert call(ws.data_ptr(), need) == tk.TK_OK
    torch.cuda.synchronize()
    # the plain entry point keeps its split-H plan for these T, and agrees under the parity rule
    assert tk.make_plan(T, H, E, k, _sms())["variant"] == 2
    s0, i0 = tk.fused_topk_gating(x, w, k)
    torch.cuda.synchronize()
    ref = oracle.fused_topk_gating(wl.hidden(), wl.gate_weight(), k, want_logits=True)
    parity.check(s.cpu().numpy(), i.cpu().numpy(), ref, label="few ws")
    parity.check(s0.cpu().numpy(), i0.cpu().numpy(), ref, label="few plain")


def test_decode_workloads():
    wl = next(w for w in workloads.DECODE if w.T == 1)
    s, i, _ = run_ws(wl.hidden(), wl.gate_weight(), wl.k)
    ref = oracle.fused_topk_gating(wl.hidden(), wl.gate_weight(), wl.k, want_logits=True)
    parity.check(s, i, ref, label=wl.name)


def test_fp8_keeps_its_plain_plan():
    plan, nbytes = tk.make_plan_ws(1, 7168, 256, 8, _sms(), fp8=True)
    assert plan["variant"] == 2 and nbytes == 0


def test_right_after_a_kernel_that_writes_hidden():
    """The few-token kernel is launched as a programmatic dependent of the previous
    kernel: its loads (plain 16-byte loads, not TMA) must still see what that
    kernel wrote -- here a copy into the hidden buffer just before each call."""
    wl = workloads.RouterWorkload("few_pdl", 2, 7168, 256, 8, seed=23)
    a_bits = wl.hidden()
    b_bits = workloads.RouterWorkload(wl.name, wl.T, wl.H, wl.E, wl.k, seed=wl.seed + 100).hidden()
    w_bits = wl.gate_weight()
    a, b, w = to_device_bf16(a_bits), to_device_bf16(b_bits), to_device_bf16(w_bits)
    x = torch.empty_like(a)
    ws = tk.gating_workspace(wl.T, wl.H, wl.E, wl.k)
    results = []
    for src in (a, b, a, b):
        x.copy_(src)
        s, i = tk.fused_topk_gating(x, w, wl.k, workspace=ws)
        results.append((s.clone(), i.clone()))
    torch.cuda.synchronize()
    for bits, (s, i) in zip((a_bits, b_bits, a_bits, b_bits), results):
        ref = oracle.fused_topk_gating(bits, w_bits, wl.k, want_logits=True)
        parity.check(s.cpu().numpy(), i.cpu().numpy(), ref, label=wl.name)


@pytest.mark.parametrize("T,E,k", [(1, 256, 8), (4, 64, 8), (3, 200, 32), (2, 16, 16)])
def test_zero_gate_gives_uniform_scores(T, E, k):
    """Every logit is 0: all ties, so the ids are 0..k-1 (lower index first) and the
    scores 1/k -- the tie order across lanes, lane merges and expert blocks."""
    H = 2048
    x = workloads.normal_bf16(5, 1, 0, T * H).reshape(T, H)
    w = np.zeros((H, E), dtype=np.uint16)
    s, i, L = run_ws(x, w, k, logits=True)
    assert np.all(L == 0.0)
    assert np.array_equal(i, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    assert np.all(np.abs(s - 1.0 / k) <= 1e-7)


@pytest.mark.parametrize("T,E", [(1, 16), (4, 32), (2, 24)])
def test_k_equals_E_full_softmax(T, E):
    """k = E: every expert is selected, in logit order; the scores are the softmax
    over all E logits."""
    wl = workloads.RouterWorkload(f"few_kE_{T}_{E}", T, 1024, E, E, seed=40 + E)
    s, i, L = run_ws(wl.hidden(), wl.gate_weight(), E, logits=True)
    ref = oracle.fused_topk_gating(wl.hidden(), wl.gate_weight(), E, want_logits=True)
    parity.check(s, i, ref, label=wl.name)
    assert np.array_equal(np.sort(i, axis=1), np.tile(np.arange(E, dtype=np.int32), (T, 1)))
