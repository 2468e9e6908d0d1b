"""FP8 (E4M3) gating on the GPU against the FP8 oracle, under the parity rule of
tests/parity.py.  Inputs: the workloads' bf16 values quantized per token
(hidden) and per expert (gate, expert-major) by torch on the CPU -- the same
bits and scales feed both sides.  Covers split-H clusters and CTA pairs,
half tiles, 512 experts, k up to 32, exact ties (duplicated experts quantize
identically), the 65536 x 7168 launches on every row, and a zero gate."""
import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def clean_error_word():
    assert torch.cuda.is_available()
    tk.device_error(clear=True)
    yield
    assert tk.device_error(clear=True) == 0, "a kernel wait expired during the GPU tests"


def run_fp8(xq, xs, wq, ws, k):
    dev = torch.device("cuda")
    args = [torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in (xq, xs, wq, ws)]
    s, i = tk.fused_topk_gating_fp8(*args, k)
    torch.cuda.synchronize()
    return s.cpu().numpy(), i.cpu().numpy()


def check_fp8(wl, duplicate_pairs=(), rows=None):
    xq, xs, wq, ws = workloads.fp8_inputs(wl)
    s, i = run_fp8(xq, xs, wq, ws, wl.k)
    if rows is None:
        ref = oracle.fused_topk_gating_fp8(xq, xs, wq, ws, wl.k, want_logits=True)
        return parity.check(s, i, ref, duplicate_pairs=duplicate_pairs, label=f"fp8-{wl.name}")
    ref = oracle.fused_topk_gating_fp8(xq[rows], xs[rows], wq, ws, wl.k, want_logits=True)
    return parity.check(s, i, ref, rows=rows, duplicate_pairs=duplicate_pairs, label=f"fp8-{wl.name}")


@pytest.mark.parametrize("T,H,E,k", [
    (64, 512, 16, 2), (1, 7168, 256, 8), (128, 7168, 256, 8), (4096, 7168, 256, 8), (300, 528, 40, 3),
    (20000, 512, 256, 8), (19999, 512, 200, 8), (16384, 4096, 64, 6), (30000, 256, 512, 32), (1000, 1024, 512, 16),
    (3, 2048, 64, 4), (129, 144, 24, 5), (200, 512, 1024, 8), (20000, 256, 768, 8), (300, 256, 1024, 32),
    (24000, 128, 1016, 32),
    # eight epilogue warps: one CTA per tile (E <= 64, k = 16) and pairs with half tiles (k = 16)
    (20000, 512, 64, 16), (40000, 512, 256, 16),
])
def test_fp8_shapes(T, H, E, k):
    check_fp8(workloads.RouterWorkload(f"fp8_{T}_{H}_{E}_{k}", T, H, E, k, seed=7))


def test_fp8_skew_ties():
    info = check_fp8(workloads.SKEW, duplicate_pairs=workloads.SKEW.duplicate_pairs)
    assert info["rows"] == workloads.SKEW.T


def test_fp8_train_all_rows():
    info = check_fp8(workloads.TRAIN)
    assert info["rows"] == workloads.TRAIN.T


def test_fp8_large_e_all_rows():
    info = check_fp8(workloads.LARGE_E)
    assert info["rows"] == workloads.LARGE_E.T


def test_fp8_zero_gate_gives_uniform_scores():
    T, H, E, k = 300, 256, 64, 8
    xq, xs = workloads.quantize_e4m3_rows(np.random.default_rng(1).standard_normal((T, H)).astype(np.float32))
    wq = np.zeros((E, H), dtype=np.uint8)
    ws = np.ones(E, dtype=np.float32)
    s, i = run_fp8(xq, xs, wq, ws, k)
    assert np.array_equal(i, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    assert np.all(np.abs(s - 1.0 / k) <= 1e-7)
