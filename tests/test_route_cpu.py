"""Host logic of the routing-metadata entry point (no kernel is launched):
argument validation before any CUDA call, and the launch plan -- every
assignment falls in exactly one warp range, at most one CTA per SM, the
workspace holds one counts row per CTA, and one CTA needs none."""
import ctypes

import pytest

import moe_router_gating_b200 as tk
from moe_router_gating_b200 import build as tkbuild


@pytest.fixture(scope="module", autouse=True)
def built():
    tkbuild.build()


@pytest.mark.parametrize("T,k,E", [(0, 8, 256), (1, 1, 1), (1, 8, 256), (4096, 8, 256), (16384, 6, 64),
                                   (65536, 8, 256), (12345, 7, 999), (3001, 16, 1024), (2**27, 8, 256)])
@pytest.mark.parametrize("num_sms", [1, 7, 148])
def test_plan_covers_every_slot_once(T, k, E, num_sms):
    p = tk.route_plan(T, k, E, num_sms)
    n = T * k
    L = p["warp_slots"]
    assert L % 32 == 0 and L >= 128
    assert 1 <= p["ctas"] <= max(1, num_sms)
    warps = p["ctas"] * (p["threads"] // 32)
    # ranges [w*L, (w+1)*L) clipped to n: they cover [0, n) iff warps*L >= n, and
    # no CTA is idle iff (ctas-1) CTAs fall short of n
    assert warps * L >= n
    assert n == 0 or (p["ctas"] - 1) * (p["threads"] // 32) * L < n
    assert p["workspace_bytes"] == (p["ctas"] * ((E + 3) // 4 * 4) * 4 if p["ctas"] > 1 else 0)
    assert p["count_smem_bytes"] <= 227 * 1024 and p["scatter_smem_bytes"] <= 227 * 1024


def test_plan_single_kernel_up_to_4096_assignments():
    assert tk.route_plan(512, 8, 256)["ctas"] == 1 and tk.route_plan(512, 8, 256)["workspace_bytes"] == 0
    assert tk.route_plan(4096, 1, 16)["ctas"] == 1
    assert tk.route_plan(4097, 1, 16)["ctas"] == 2


def test_plan_workspace_bound_on_b200():
    # the header's stated bound: at most 148 x 1024 x 4 bytes
    assert tk.route_plan(2**31 // 16 - 1, 16, 1024, 148)["workspace_bytes"] == 148 * 1024 * 4


@pytest.mark.parametrize("T,k,E,code", [
    (-1, 8, 256, tk.TK_ERR_INVALID_ARG), (4, 0, 256, tk.TK_ERR_INVALID_ARG), (4, 8, 0, tk.TK_ERR_INVALID_ARG),
    (4, 8, 1025, tk.TK_ERR_UNSUPPORTED), (2**28, 8, 256, tk.TK_ERR_UNSUPPORTED),
])
def test_plan_rejects(T, k, E, code):
    with pytest.raises(tk.TkGatingError) as ei:
        tk.route_plan(T, k, E)
    assert ei.value.status == code


def test_route_rejects_before_any_cuda_call():
    lib = tk.library()
    buf = (ctypes.c_int32 * 64)()
    a = ctypes.addressof(buf)
    assert lib.tk_gating_route(a, -1, 8, 16, a, a, a, None) == tk.TK_ERR_INVALID_ARG
    assert lib.tk_gating_route(a, 4, 8, 2000, a, a, a, None) == tk.TK_ERR_UNSUPPORTED
    assert lib.tk_gating_route(a, 4, 2, 16, None, a, a, None) == tk.TK_ERR_INVALID_ARG   # offsets NULL
    assert lib.tk_gating_route(None, 4, 2, 16, a, a, a, None) == tk.TK_ERR_INVALID_ARG   # ids NULL, n > 0
    assert lib.tk_gating_route(a, 4, 2, 16, a, None, a, None) == tk.TK_ERR_INVALID_ARG
    assert lib.tk_gating_route(a + 2, 4, 2, 16, a, a, a, None) == tk.TK_ERR_ALIGNMENT
    assert lib.tk_gating_route(a, 4, 2, 16, a, a + 1, a, None) == tk.TK_ERR_ALIGNMENT
