"""Parity on the GPU for more than 256 experts (two MMA chunks of at most 256
experts each) and for up to 32 selected experts, against the CPU oracle under
the rule of tests/parity.py.  Covers both kernel families (split-H clusters
for few tokens, CTA pairs with a single-buffered accumulator for many), pair
half tiles, E padding inside the second chunk, and exact ties across the
chunk boundary and across the halves a pair's CTAs hold."""
import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import oracle
import parity
import workloads
from gpu_helpers import check_against_oracle, check_workload, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def clean_error_word():
    assert torch.cuda.is_available()
    tk.device_error(clear=True)
    yield
    assert tk.device_error(clear=True) == 0, "a kernel wait expired during the GPU tests"


@pytest.mark.parametrize("T,H,E,k", [
    # split-H clusters
    (1, 7168, 512, 8), (7, 1024, 512, 32), (128, 2048, 320, 16), (1000, 1024, 512, 32), (4096, 1024, 384, 8),
    (129, 512, 264, 1), (300, 520, 504, 17),
    # CTA pairs, two chunks, single accumulator (and half tiles: T just above a full round)
    (20000, 512, 512, 8), (30000, 512, 320, 32), (19999, 256, 448, 5), (40000, 128, 264, 3),
    # two expert groups of up to 512 (E up to 1024), split-H and pairs
    (1, 7168, 1024, 8), (100, 1024, 640, 32), (4096, 512, 1024, 8), (20000, 256, 1024, 8), (30000, 256, 776, 16),
    (300, 256, 1024, 32), (24000, 128, 1016, 32),
    # k up to 32 with one chunk
    (2000, 1024, 256, 32), (40000, 512, 256, 32), (5000, 256, 64, 32), (700, 256, 32, 32),
    # one CTA per 128-token tile (E <= 64) with eight epilogue warps (lists of 16 and 32)
    (20000, 512, 64, 16), (20011, 512, 64, 32), (12000, 256, 48, 24),
])
def test_large_expert_shapes(T, H, E, k):
    check_workload(workloads.RouterWorkload(f"large_{T}_{H}_{E}_{k}", T, H, E, k, seed=5))


@pytest.mark.parametrize("T", [300, 24000])
def test_ties_across_chunk_and_half_boundaries(T):
    # equal gate columns give equal logits: the lower expert index must win,
    # whichever chunk, pair half or CTA holds the other copy
    E, H, k = 512, 512, 8
    wl = workloads.RouterWorkload(f"ties_{T}", T, H, E, k, seed=13)
    w = wl.gate_weight().copy()
    pairs = ((255, 256), (127, 128), (383, 384), (0, 511), (300, 301), (64, 448))
    for a, b in pairs:
        w[:, b] = w[:, a]
    # make the tied columns competitive: scale them up
    for a, b in pairs:
        w[:, a] = workloads.round_bf16(workloads.bf16_to_f64(w[:, a]) * 3.0)
        w[:, b] = w[:, a]
    check_against_oracle(wl.hidden(), w, k, duplicate_pairs=pairs, label=f"ties_{T}")


@pytest.mark.parametrize("T", [300, 24000])
def test_ties_across_expert_groups(T):
    # experts 511 and 512 sit in different groups (computed one after the other):
    # equal logits must still go to the lower index
    E, H, k = 1024, 256, 8
    wl = workloads.RouterWorkload(f"gties_{T}", T, H, E, k, seed=17)
    w = wl.gate_weight().copy()
    pairs = ((511, 512), (0, 1023), (300, 700), (255, 256))
    for a, b in pairs:
        w[:, a] = workloads.round_bf16(workloads.bf16_to_f64(w[:, a]) * 3.0)
        w[:, b] = w[:, a]
    check_against_oracle(wl.hidden(), w, k, duplicate_pairs=pairs, label=f"gties_{T}")


def test_large_e_workload_all_rows():
    """The 65536 x 7168 x 512 launch the benchmark times, every row against the oracle."""
    wl = workloads.LARGE_E
    info = check_workload(wl)
    assert info["rows"] == wl.T


def test_e1024_workload_all_rows():
    """65536 x 7168 x 1024: two expert groups per tile, every row against the oracle."""
    wl = workloads.E1024
    info = check_workload(wl)
    assert info["rows"] == wl.T


def test_large_k_workload():
    check_workload(workloads.LARGE_K)
