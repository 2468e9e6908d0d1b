"""The logits the kernels rank, measured against the oracle's fp64 logits.

The verification entry points (tk_gating_fused_topk_logits and its FP8 twin)
run the same launch as the plain call and also store every fp32 logit the
selection saw.  On every row of each workload this checks

* the error budget: max |logit_gpu - logit_oracle| <= parity.LOGIT_ATOL
  (the logits step of the naive form, ``hidden_states @ gate_weight``, on the
  chenxutan.com page "TileKernels 深度解析", section 4.1);
* the selection and softmax on the kernel's own fp32 logits, exactly: ids are
  the top-k under (value descending, index ascending), scores their softmax;
* that asking for the logits changes nothing: scores and ids are bitwise those
  of the plain call;
* for duplicated gate columns, bit-identical logits, whichever MMA chunk,
  CTA of a pair, split-H owner or expert group computed each copy.

The measured errors are printed (``-s``) and recorded in the design notes.
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


def gpu_with_logits(x_bits, w_bits, k):
    x, w = to_device_bf16(x_bits), to_device_bf16(w_bits)
    T, E = x_bits.shape[0], w_bits.shape[1]
    logits = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    s, i = tk.fused_topk_gating(x, w, k, logits=logits)
    s0, i0 = tk.fused_topk_gating(x, w, k)
    torch.cuda.synchronize()
    assert torch.equal(s, s0) and torch.equal(i, i0), "the logits call changed scores or ids"
    return s.cpu().numpy(), i.cpu().numpy(), logits.cpu().numpy()


def check_logits(x_bits, w_bits, k, label, duplicate_pairs=()):
    s, i, L = gpu_with_logits(x_bits, w_bits, k)
    assert not np.isnan(L).any(), f"{label}: a logit was not stored"
    ref = oracle.fused_topk_gating(x_bits, w_bits, k, want_logits=True)
    err = parity.logit_error(L, ref.logits)
    print(f"\n{label}: T={x_bits.shape[0]} H={x_bits.shape[1]} E={w_bits.shape[1]} max |logit error| = {err:.3e}")
    assert err <= parity.LOGIT_ATOL, f"{label}: logit error {err}"
    parity.check_own_selection(s, i, L, label=label)
    for a, b in duplicate_pairs:
        assert np.array_equal(L[:, a].view(np.uint32), L[:, b].view(np.uint32)), \
            f"{label}: duplicated columns {a}, {b} gave different logits"
    parity.check(s, i, ref, duplicate_pairs=duplicate_pairs, label=label)
    return err


@pytest.mark.parametrize("name", ["tiny", "deepseek", "skew", "train", "decode_T1", "decode_T8", "decode_T32",
                                  "decode_T128", "decode_T256", "large_e", "large_k", "e1024"])
def test_logit_error_budget(name):
    wl = workloads.WORKLOADS[name]
    check_logits(wl.hidden(), wl.gate_weight(), wl.k, name, duplicate_pairs=wl.duplicate_pairs)


@pytest.mark.parametrize("T,H,E,k", [
    (2048, 512, 64, 8),      # split-H owners
    (24000, 512, 256, 8),    # CTA pairs: copies in the two CTAs' gate halves, half tiles
    (24000, 512, 512, 8),    # two MMA chunks
    (300, 256, 1024, 8),     # two expert groups, split-H
    (24000, 256, 1024, 8),   # two expert groups, pairs
    (20000, 512, 48, 4),     # one CTA per tile
])
def test_duplicated_columns_give_identical_logits(T, H, E, k):
    wl = workloads.RouterWorkload(f"dup_{T}_{E}", T, H, E, k, seed=19)
    w = wl.gate_weight().copy()
    # disjoint pairs: both ends of the expert range, the middle (CTA pair halves,
    # or the expert-group boundary 511 | 512), a quarter apart, and for more than
    # 512 experts the MMA chunk boundary 255 | 256 inside group 0
    pairs = [(0, E - 1), (1, 2), (E // 2 - 1, E // 2), (E // 4 - 1, 3 * E // 4)]
    if E > 512:
        pairs.append((254, 256))
    pairs = tuple(sorted(pairs))
    flat = [c for pr in pairs for c in pr]
    assert len(flat) == len(set(flat)), "a column in two pairs would not stay a copy"
    for a, b in pairs:  # scaled up so that the copies are often selected
        w[:, a] = workloads.round_bf16(workloads.bf16_to_f64(w[:, a]) * 3.0)
        w[:, b] = w[:, a]
    check_logits(wl.hidden(), w, k, f"dup_{T}_{H}_{E}_{k}", duplicate_pairs=pairs)


@pytest.mark.parametrize("name", ["tiny", "deepseek", "skew", "train", "decode_T1", "large_k"])
def test_fp8_logit_error_budget(name):
    wl = workloads.WORKLOADS[name]
    xq, xs, wq, ws = workloads.fp8_inputs(wl)
    dev = [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in (xq, xs, wq, ws)]
    logits = torch.full((wl.T, wl.E), float("nan"), dtype=torch.float32, device="cuda")
    s, i = tk.fused_topk_gating_fp8(*dev, wl.k, logits=logits)
    s0, i0 = tk.fused_topk_gating_fp8(*dev, wl.k)
    torch.cuda.synchronize()
    assert torch.equal(s, s0) and torch.equal(i, i0)
    L = logits.cpu().numpy()
    ref = oracle.fused_topk_gating_fp8(xq, xs, wq, ws, wl.k, want_logits=True)
    err = parity.logit_error(L, ref.logits)
    print(f"\nfp8-{name}: max |logit error| = {err:.3e}")
    assert err <= parity.LOGIT_ATOL
    s, i = s.cpu().numpy(), i.cpu().numpy()
    parity.check_own_selection(s, i, L, label=f"fp8-{name}")
    for a, b in wl.duplicate_pairs:
        assert np.array_equal(L[:, a].view(np.uint32), L[:, b].view(np.uint32))
    parity.check(s, i, ref, duplicate_pairs=wl.duplicate_pairs, label=f"fp8-{name}")
