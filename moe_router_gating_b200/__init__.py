"""Fused MoE top-k gating on NVIDIA B200 (sm_100a).

``fused_topk_gating(hidden, gate_weight, top_k)`` computes, in one kernel launch,
``softmax(topk(hidden @ gate_weight, k))`` as the chenxutan.com page describes
TileKernels' gating (section 4.1 "MoE Gating"): logits are accumulated in fp32
on the tensor cores and never written to global memory; only the fp32 scores
and int32 expert ids are.

This package is a thin ctypes binding of the in-tree CUDA library
``libtk_gating.so`` (C ABI in ``include/tk_gating.h``).  PyTorch supplies device
memory and streams; every step of the computation runs in the library's
kernels.  There is no CPU fallback: without the built library the import of
the binding fails, and without an sm_100 device the calls raise.
"""
from ._binding import (  # noqa: F401
    TK_OK,
    TK_ERR_ALIGNMENT,
    TK_ERR_CUDA,
    TK_ERR_DEVICE_TIMEOUT,
    TK_ERR_INVALID_ARG,
    TK_ERR_UNSUPPORTED,
    TkGatingError,
    clock_counters,
    device_error,
    exported_symbols,
    fused_topk_gating,
    fused_topk_gating_fp8,
    fused_topk_gating_fp8_ptr,
    fused_topk_gating_host,
    fused_topk_gating_ptr,
    fused_topk_gating_route,
    fused_topk_gating_route_ptr,
    fused_topk_gating_ws_ptr,
    gating_workspace,
    library,
    library_path,
    make_plan,
    make_plan_ws,
    route,
    route_plan,
    route_ptr,
    route_workspace,
    route_static_ptr,
    set_wait_timeout_ns,
    status_string,
    workspace_bytes,
)

__all__ = [
    "fused_topk_gating", "fused_topk_gating_fp8", "fused_topk_gating_host", "fused_topk_gating_ptr",
    "fused_topk_gating_route", "fused_topk_gating_route_ptr", "route_workspace", "make_plan", "route", "route_plan",
    "fused_topk_gating_ws_ptr", "gating_workspace", "workspace_bytes", "make_plan_ws",
    "route_ptr", "route_static_ptr", "device_error", "clock_counters",
    "set_wait_timeout_ns", "status_string", "TkGatingError", "library", "library_path",
]
