"""Helpers shared by the GPU tests: run the CUDA path on seeded inputs and
compare with the oracle under the parity rule."""
from __future__ import annotations

import numpy as np
import torch

import moe_router_gating_b200 as tk
import oracle
import parity
import workloads


def to_device_bf16(bits: np.ndarray) -> torch.Tensor:
    return workloads.to_torch_bf16(bits).cuda()


def run_gpu(x_bits: np.ndarray, w_bits: np.ndarray, k: int):
    x = to_device_bf16(x_bits)
    w = to_device_bf16(w_bits)
    scores, ids = tk.fused_topk_gating(x, w, k)
    torch.cuda.synchronize()
    return scores.cpu().numpy(), ids.cpu().numpy()


def check_against_oracle(x_bits, w_bits, k, duplicate_pairs=(), label=""):
    s, i = run_gpu(x_bits, w_bits, k)
    ref = oracle.fused_topk_gating(x_bits, w_bits, k, want_logits=True)
    return parity.check(s, i, ref, duplicate_pairs=duplicate_pairs, label=label)


def check_workload(wl: workloads.RouterWorkload, label=None):
    return check_against_oracle(wl.hidden(), wl.gate_weight(), wl.k, wl.duplicate_pairs, label or wl.name)
