"""Every wait in the kernels is bounded: an expired wait is reported through the
device error word, the kernel stops (its own copies and MMAs drained), and the
CUDA context stays usable.  The wait is made to run out by setting a 1 us
limit, far shorter than one tile's MMAs (about 30 us at H = 7168); no fault,
trap or hang is involved.  Every kernel family is covered: the one-CTA row
tiles, the CTA pairs (whose CTAs wait on each other's barriers, and whose
epilogue warps agree on each tile before the half tiles' list exchange) and the
split-H clusters (cluster barriers after an abort; expert groups skipped)."""
import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import oracle
import parity
import workloads
from gpu_helpers import to_device_bf16

pytestmark = pytest.mark.gpu


# (T, H, E, k, planned variant): every kernel family, including the CTA pairs'
# balanced last round of half tiles (their list exchange is the one place where
# the epilogue warps of a CTA wait for one another) and the split-H clusters
# with one and with two expert groups.  H is large for split-H so that each
# CTA's mainloop outlasts a polling interval of the waits (20 us).
ABORT_CASES = [
    (20000, 7168, 64, 4, 1),     # one CTA per 128-token tile
    (20000, 7168, 256, 8, 3),    # CTA pairs: 74 full tiles, then 9 half tiles
    (20000, 4096, 1024, 8, 3),   # CTA pairs, two expert groups per tile
    (4096, 32768, 256, 8, 2),    # split-H, clusters of 4
    (128, 32768, 256, 8, 2),     # split-H, one cluster of 16
    (128, 32768, 1024, 8, 2),    # split-H, two expert groups
]


@pytest.mark.parametrize("T,H,E,k,variant", ABORT_CASES)
def test_expired_wait_is_reported_and_context_survives(T, H, E, k, variant):
    wl = workloads.RouterWorkload(f"bounded_{T}_{H}_{E}", T, H, E, k, seed=8)
    assert tk.make_plan(wl.T, wl.H, wl.E, wl.k)["variant"] == variant
    x_bits, w_bits = wl.hidden(), wl.gate_weight()
    x, w = to_device_bf16(x_bits), to_device_bf16(w_bits)
    tk.device_error(clear=True)

    tk.set_wait_timeout_ns(1000)
    try:
        tk.fused_topk_gating(x, w, wl.k)  # the launch itself succeeds
        torch.cuda.synchronize()
    finally:
        tk.set_wait_timeout_ns(1_000_000_000)
    word = tk.device_error(clear=True)
    assert word != 0, "a 1 us wait limit must expire during this launch"

    # same context, default limit: correct results and a clean error word
    s, i = tk.fused_topk_gating(x, w, wl.k)
    torch.cuda.synchronize()
    assert tk.device_error(clear=True) == 0
    rows = np.unique(np.concatenate([np.arange(0, wl.T, max(1, wl.T // 150)), [wl.T - 1]]))
    ref = oracle.fused_topk_gating(x_bits[rows], w_bits, wl.k, want_logits=True)
    parity.check(s.cpu().numpy(), i.cpu().numpy(), ref, rows=rows, label="after-timeout")


def test_timeout_setter_rejects_tiny_limits():
    with pytest.raises(tk.TkGatingError):
        tk.set_wait_timeout_ns(10)
