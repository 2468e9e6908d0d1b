"""Every wait in the kernels is bounded: an expired wait is reported through the
device error word, the kernel stops (its own copies and MMAs drained), and the
CUDA context stays usable.  The wait is made to run out by setting a 1 us
limit, far shorter than one tile's MMAs (about 30 us at H = 7168); no fault,
trap or hang is involved."""
import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import oracle
import parity
import workloads
from gpu_helpers import to_device_bf16

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives():
    # many tiles, E <= 64: the persistent one-CTA-per-tile kernel
    wl = workloads.RouterWorkload("bounded", 20000, 7168, 64, 4, seed=8)
    assert tk.make_plan(wl.T, wl.H, wl.E, wl.k)["variant"] == 1
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
    assert word != 0, "a 1 us wait limit must expire during a 20000-token launch"

    # same context, default limit: correct results and a clean error word
    s, i = tk.fused_topk_gating(x, w, wl.k)
    torch.cuda.synchronize()
    assert tk.device_error(clear=True) == 0
    rows = np.arange(0, wl.T, 97)
    ref = oracle.fused_topk_gating(x_bits[rows], w_bits, wl.k, want_logits=True)
    parity.check(s.cpu().numpy(), i.cpu().numpy(), ref, rows=rows, label="after-timeout")


def test_timeout_setter_rejects_tiny_limits():
    with pytest.raises(tk.TkGatingError):
        tk.set_wait_timeout_ns(10)
