"""ctypes marshalling for libtk_gating.so (argument checks and pointers only)."""
from __future__ import annotations

import ctypes
import os
import re
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_PKG)
HEADER = os.path.join(_ROOT, "include", "tk_gating.h")
# TK_GATING_DEBUG=1 in the environment selects the build with the kernels' index
# checks compiled in (python -m moe_router_gating_b200.build --debug)
_LIB_PATH = os.path.join(_PKG, "libtk_gating_debug.so" if os.environ.get("TK_GATING_DEBUG", "0") not in ("", "0")
                         else "libtk_gating.so")

TK_OK = 0
TK_ERR_INVALID_ARG = -1
TK_ERR_UNSUPPORTED = -2
TK_ERR_ALIGNMENT = -3
TK_ERR_CUDA = -4
TK_ERR_DEVICE_TIMEOUT = -5

_lock = threading.Lock()
_lib = None


class TkGatingError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} ({status})")
        self.status = status


class _Plan(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "variant", "block_m", "n_pad", "num_tiles", "k_blocks", "split_h", "stages", "grid", "cluster",
        "threads", "smem_bytes", "tmem_cols", "num_half_tiles", "slices_per_stage", "expert_groups",
        "num_split_tiles", "split_k_block", "h_rows")]


class _RoutePlan(ctypes.Structure):
    _fields_ = [("ctas", ctypes.c_int32), ("threads", ctypes.c_int32), ("warp_slots", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_int64), ("count_smem_bytes", ctypes.c_int32),
                ("scatter_smem_bytes", ctypes.c_int32), ("fused_workspace_bytes", ctypes.c_int64)]


def library_path() -> str:
    return _LIB_PATH


def library() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                                   "`python -m moe_router_gating_b200.build` (add --debug for the checked build; "
                                   "needs nvcc)")
            lib = ctypes.CDLL(_LIB_PATH)
            vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
            lib.tk_gating_fused_topk.argtypes = [vp, vp, i64, i64, i64, i32, vp, vp, vp]
            lib.tk_gating_fused_topk.restype = ctypes.c_int
            lib.tk_gating_fused_topk_host.argtypes = [vp, vp, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp]
            lib.tk_gating_fused_topk_host.restype = ctypes.c_int
            lib.tk_gating_fused_topk_fp8.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, vp, vp, vp]
            lib.tk_gating_fused_topk_fp8.restype = ctypes.c_int
            lib.tk_gating_fused_topk_route.argtypes = [vp, vp, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, i64, vp]
            lib.tk_gating_fused_topk_route.restype = ctypes.c_int
            lib.tk_gating_fused_topk_ws.argtypes = [vp, vp, i64, i64, i64, i32, vp, vp, vp, i64, vp]
            lib.tk_gating_fused_topk_ws.restype = ctypes.c_int
            lib.tk_gating_fused_topk_ws_logits.argtypes = [vp, vp, i64, i64, i64, i32, vp, vp, vp, vp, i64, vp]
            lib.tk_gating_fused_topk_ws_logits.restype = ctypes.c_int
            lib.tk_gating_fused_topk_fp8_ws.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, vp, vp, vp, i64, vp]
            lib.tk_gating_fused_topk_fp8_ws.restype = ctypes.c_int
            lib.tk_gating_make_plan_ws.argtypes = [i64, i64, i64, i32, i32, ctypes.POINTER(_Plan),
                                                   ctypes.POINTER(ctypes.c_int64)]
            lib.tk_gating_make_plan_ws.restype = ctypes.c_int
            lib.tk_gating_make_plan_fp8_ws.argtypes = lib.tk_gating_make_plan_ws.argtypes
            lib.tk_gating_make_plan_fp8_ws.restype = ctypes.c_int
            lib.tk_gating_workspace_bytes.argtypes = [i64, i64, i64, i32, i32, ctypes.POINTER(ctypes.c_int64)]
            lib.tk_gating_workspace_bytes.restype = ctypes.c_int
            lib.tk_gating_fused_topk_logits.argtypes = [vp, vp, i64, i64, i64, i32, vp, vp, vp, vp]
            lib.tk_gating_fused_topk_logits.restype = ctypes.c_int
            lib.tk_gating_fused_topk_fp8_logits.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, vp, vp, vp, vp]
            lib.tk_gating_fused_topk_fp8_logits.restype = ctypes.c_int
            u64p = ctypes.POINTER(ctypes.c_uint64)
            lib.tk_gating_clock_counters.argtypes = [u64p, u64p, u64p, i32]
            lib.tk_gating_clock_counters.restype = ctypes.c_int
            lib.tk_gating_make_plan.argtypes = [i64, i64, i64, i32, i32, ctypes.POINTER(_Plan)]
            lib.tk_gating_make_plan.restype = ctypes.c_int
            lib.tk_gating_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
            lib.tk_gating_device_error.restype = ctypes.c_int
            lib.tk_gating_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
            lib.tk_gating_set_wait_timeout_ns.restype = ctypes.c_int
            lib.tk_gating_route.argtypes = [vp, i64, i32, i32, vp, vp, vp, vp]
            lib.tk_gating_route.restype = ctypes.c_int
            lib.tk_gating_route_static.argtypes = [vp, i64, i32, i32, vp, vp, vp, vp]
            lib.tk_gating_route_static.restype = ctypes.c_int
            lib.tk_gating_route_plan.argtypes = [i64, i32, i32, i32, ctypes.POINTER(_RoutePlan)]
            lib.tk_gating_route_plan.restype = ctypes.c_int
            lib.tk_gating_status_string.argtypes = [ctypes.c_int]
            lib.tk_gating_status_string.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def exported_symbols() -> list[str]:
    """Function names declared in include/tk_gating.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*TK_API\s+(?:const\s+)?\w+\s*\*?\s*(tk_gating_\w+)\s*\(", text, re.M)))


def status_string(status: int) -> str:
    return library().tk_gating_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != TK_OK:
        raise TkGatingError(status, where)


def _stream_handle(stream, device) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream)


def fused_topk_gating_ptr(hidden: int, gate_weight: int, T: int, H: int, E: int, k: int, scores: int, ids: int,
                          stream: int = 0) -> int:
    """Raw C-ABI call with integer device pointers; returns the tk_status."""
    return int(library().tk_gating_fused_topk(hidden, gate_weight, T, H, E, k, scores, ids, stream))


def fused_topk_gating_ws_ptr(hidden: int, gate_weight: int, T: int, H: int, E: int, k: int, scores: int, ids: int,
                             workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    """Raw C-ABI call of the workspace entry point (integer device pointers);
    returns the tk_status."""
    return int(library().tk_gating_fused_topk_ws(hidden, gate_weight, T, H, E, k, scores, ids, workspace,
                                                 workspace_bytes, stream))


def workspace_bytes(T: int, H: int, E: int, k: int, fp8: bool = False) -> int:
    """Bytes of workspace the workspace entry points need for (T, H, E, k) on the
    current device (0 where they make the launch without one)."""
    n = ctypes.c_int64(0)
    _check(library().tk_gating_workspace_bytes(T, H, E, k, 1 if fp8 else 0, ctypes.byref(n)),
           "tk_gating_workspace_bytes")
    return int(n.value)


def gating_workspace(T: int, H: int, E: int, k: int, device=None, fp8: bool = False):
    """A zeroed uint8 CUDA tensor (at least 256 bytes) to serve as the
    ``workspace`` of ``fused_topk_gating`` / ``fused_topk_gating_fp8`` for
    (T, H, E, k) on ``device``; every call leaves it ready for the next one on
    the same stream.  Calls that may overlap on the device need their own."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        n = workspace_bytes(T, H, E, k, fp8)
    return torch.zeros(max(256, n), dtype=torch.uint8, device=dev)


def make_plan_ws(T: int, H: int, E: int, k: int, num_sms: int = 148, fp8: bool = False) -> tuple[dict, int]:
    """The launch of the workspace entry point (fp8: of the FP8 one, H in FP8 values) and its
    workspace bytes (host logic only)."""
    p = _Plan()
    n = ctypes.c_int64(0)
    fn = library().tk_gating_make_plan_fp8_ws if fp8 else library().tk_gating_make_plan_ws
    _check(fn(T, H, E, k, num_sms, ctypes.byref(p), ctypes.byref(n)),
           "tk_gating_make_plan_fp8_ws" if fp8 else "tk_gating_make_plan_ws")
    return {name: getattr(p, name) for name, _ in _Plan._fields_}, int(n.value)


def _check_workspace(workspace, device) -> None:
    if not workspace.is_cuda or workspace.device != device or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor on the inputs' device")


def fused_topk_gating(hidden, gate_weight, top_k: int, scores=None, ids=None, stream=None, logits=None,
                      workspace=None):
    """``(scores[T,k] fp32, ids[T,k] int32) = softmax(topk(hidden @ gate_weight))``.

    ``hidden`` is a CUDA bf16 ``[T, H]`` tensor and ``gate_weight`` a CUDA bf16
    ``[H, E]`` tensor, both contiguous.  Output tensors may be passed in.  The
    launch goes on ``stream`` (default: the current torch stream).  Passing a
    contiguous fp32 ``[T, E]`` CUDA tensor as ``logits`` calls the verification
    entry point, which also stores every logit the selection ranked.  Passing a
    ``workspace`` (from ``gating_workspace``) calls the workspace entry point,
    whose last round of a many-token launch splits its tiles in H between CTA
    pairs.
    """
    import torch
    if hidden.dtype != torch.bfloat16 or gate_weight.dtype != torch.bfloat16:
        raise TypeError("hidden and gate_weight must be torch.bfloat16")
    if hidden.dim() != 2 or gate_weight.dim() != 2 or hidden.shape[1] != gate_weight.shape[0]:
        raise ValueError(f"shapes {tuple(hidden.shape)} @ {tuple(gate_weight.shape)} do not chain")
    if not hidden.is_cuda or not gate_weight.is_cuda or hidden.device != gate_weight.device:
        raise ValueError("hidden and gate_weight must be CUDA tensors on one device")
    if not hidden.is_contiguous() or not gate_weight.is_contiguous():
        raise ValueError("hidden and gate_weight must be contiguous (row-major)")
    T, H = hidden.shape
    E = gate_weight.shape[1]
    if scores is None:
        scores = torch.empty((T, top_k), dtype=torch.float32, device=hidden.device)
    if ids is None:
        ids = torch.empty((T, top_k), dtype=torch.int32, device=hidden.device)
    if scores.shape != (T, top_k) or ids.shape != (T, top_k) or scores.dtype != torch.float32 \
            or ids.dtype != torch.int32 or not scores.is_contiguous() or not ids.is_contiguous():
        raise ValueError("scores must be fp32 [T,k] and ids int32 [T,k], contiguous")
    lib = library()
    args = (hidden.data_ptr(), gate_weight.data_ptr(), T, H, E, int(top_k), scores.data_ptr(), ids.data_ptr())
    fn, name = lib.tk_gating_fused_topk, "tk_gating_fused_topk"
    if logits is not None:
        _check_logits(logits, T, E, hidden.device)
        args = args + (logits.data_ptr(),)
        fn, name = lib.tk_gating_fused_topk_logits, "tk_gating_fused_topk_logits"
    if workspace is not None:
        _check_workspace(workspace, hidden.device)
        args = args + (workspace.data_ptr(), workspace.numel() * workspace.element_size())
        fn, name = ((lib.tk_gating_fused_topk_ws_logits, "tk_gating_fused_topk_ws_logits") if logits is not None
                    else (lib.tk_gating_fused_topk_ws, "tk_gating_fused_topk_ws"))
    if hidden.device.index == torch.cuda.current_device():
        st = fn(*args, _stream_handle(stream, hidden.device))
    else:
        with torch.cuda.device(hidden.device):
            st = fn(*args, _stream_handle(stream, hidden.device))
    _check(st, name)
    return scores, ids


_route_ws_lock = threading.Lock()
_route_ws = {}  # (device index, stream handle) -> zeroed int32 workspace of fused_topk_gating_route


def route_workspace(T: int, k: int, E: int, device=None):
    """A zeroed int32 CUDA tensor large enough to serve as the workspace of
    ``fused_topk_gating_route`` for (T, k, E) on ``device`` (at least 4 elements).
    Zero it again only if a call reported bit 6 of the device error word."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    nbytes = route_plan(T, k, E, sms)["fused_workspace_bytes"]
    return torch.zeros(max(4, (nbytes + 3) // 4), dtype=torch.int32, device=dev)


def fused_topk_gating_route_ptr(hidden: int, gate_weight: int, T: int, H: int, E: int, k: int, scores: int, ids: int,
                                offsets: int, sorted_slots: int, slot_pos: int, workspace: int, workspace_bytes: int,
                                stream: int = 0) -> int:
    """Raw C-ABI call of the fused gating + routing entry point (integer device
    pointers); returns the tk_status."""
    return int(library().tk_gating_fused_topk_route(hidden, gate_weight, T, H, E, k, scores, ids, offsets,
                                                    sorted_slots, slot_pos, workspace, workspace_bytes, stream))


def fused_topk_gating_route(hidden, gate_weight, top_k: int, workspace=None, stream=None):
    """Gating and the routing metadata of its ids in one call, the counts per
    expert taken by the gating kernel: ``(scores, ids, offsets, sorted_slots,
    slot_pos)``, the results of ``fused_topk_gating`` and then ``route``.

    ``workspace`` (int32 CUDA tensor, zero before its first use, left zero by
    every call) defaults to one the binding keeps per device and stream; pass
    one of ``route_workspace``'s when capturing the call into a CUDA graph."""
    import torch
    if hidden.dtype != torch.bfloat16 or gate_weight.dtype != torch.bfloat16:
        raise TypeError("hidden and gate_weight must be torch.bfloat16")
    if hidden.dim() != 2 or gate_weight.dim() != 2 or hidden.shape[1] != gate_weight.shape[0]:
        raise ValueError(f"shapes {tuple(hidden.shape)} @ {tuple(gate_weight.shape)} do not chain")
    if not hidden.is_cuda or hidden.device != gate_weight.device or not hidden.is_contiguous() \
            or not gate_weight.is_contiguous():
        raise ValueError("hidden and gate_weight must be contiguous CUDA tensors on one device")
    T, H = hidden.shape
    E = gate_weight.shape[1]
    k = int(top_k)
    dev = hidden.device
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev) if stream is None else stream
        if workspace is None:
            key = (dev.index, int(s.cuda_stream))
            sms = torch.cuda.get_device_properties(dev).multi_processor_count
            need = route_plan(T, k, E, sms)["fused_workspace_bytes"]
            with _route_ws_lock:
                workspace = _route_ws.get(key)
                if workspace is None or workspace.numel() * 4 < need:
                    with torch.cuda.stream(s):  # zeroed in the order of the calls that use it
                        workspace = torch.zeros(max(4, (need + 3) // 4), dtype=torch.int32, device=dev)
                    _route_ws[key] = workspace
        if workspace.dtype != torch.int32 or not workspace.is_cuda or workspace.device != dev \
                or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous int32 CUDA tensor on the inputs' device")
        scores = torch.empty((T, k), dtype=torch.float32, device=dev)
        ids = torch.empty((T, k), dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        sorted_slots = torch.empty(T * k, dtype=torch.int32, device=dev)
        slot_pos = torch.empty((T, k), dtype=torch.int32, device=dev)
        st = library().tk_gating_fused_topk_route(
            hidden.data_ptr(), gate_weight.data_ptr(), T, H, E, k, scores.data_ptr(), ids.data_ptr(),
            offsets.data_ptr(), sorted_slots.data_ptr(), slot_pos.data_ptr(), workspace.data_ptr(),
            workspace.numel() * 4, int(s.cuda_stream))
    _check(st, "tk_gating_fused_topk_route")
    return scores, ids, offsets, sorted_slots, slot_pos


def _check_logits(logits, T: int, E: int, device) -> None:
    import torch
    if logits.dtype != torch.float32 or tuple(logits.shape) != (T, E) or not logits.is_contiguous() \
            or logits.device != device:
        raise ValueError(f"logits must be a contiguous fp32 [{T}, {E}] tensor on {device}")


def fused_topk_gating_fp8_ptr(hidden_q: int, hidden_scale: int, gate_q: int, gate_scale: int, T: int, H: int,
                              E: int, k: int, scores: int, ids: int, stream: int = 0) -> int:
    """Raw C-ABI call of the FP8 entry point with integer device pointers; returns the tk_status."""
    return int(library().tk_gating_fused_topk_fp8(hidden_q, hidden_scale, gate_q, gate_scale, T, H, E, k, scores,
                                                  ids, stream))


def fused_topk_gating_fp8(hidden_q, hidden_scale, gate_q, gate_scale, top_k: int, scores=None, ids=None,
                          stream=None, logits=None, workspace=None):
    """Fused gating on FP8 E4M3 inputs: ``hidden_q`` [T, H] and ``gate_q`` [E, H]
    (expert-major) as torch.float8_e4m3fn or torch.uint8 CUDA tensors, with fp32
    ``hidden_scale`` [T] and ``gate_scale`` [E].  Returns ``(scores, ids)``.
    ``logits`` (fp32 [T, E]) selects the verification entry point, which also
    stores every scaled logit the selection ranked; ``workspace`` (from
    ``gating_workspace(..., fp8=True)``) the workspace entry point (not
    combined with ``logits``)."""
    import torch
    fp8_types = (torch.float8_e4m3fn, torch.uint8)
    if hidden_q.dtype not in fp8_types or gate_q.dtype not in fp8_types:
        raise TypeError("hidden_q and gate_q must be torch.float8_e4m3fn (or their uint8 bits)")
    if hidden_scale.dtype != torch.float32 or gate_scale.dtype != torch.float32:
        raise TypeError("hidden_scale and gate_scale must be torch.float32")
    if hidden_q.dim() != 2 or gate_q.dim() != 2 or hidden_q.shape[1] != gate_q.shape[1]:
        raise ValueError(f"hidden_q {tuple(hidden_q.shape)} and gate_q {tuple(gate_q.shape)} must be [T,H] and [E,H]")
    T, H = hidden_q.shape
    E = gate_q.shape[0]
    if hidden_scale.shape != (T,) or gate_scale.shape != (E,):
        raise ValueError("hidden_scale must be [T] and gate_scale [E]")
    tensors = (hidden_q, hidden_scale, gate_q, gate_scale)
    if any(not t.is_cuda or t.device != hidden_q.device or not t.is_contiguous() for t in tensors):
        raise ValueError("inputs must be contiguous CUDA tensors on one device")
    if scores is None:
        scores = torch.empty((T, top_k), dtype=torch.float32, device=hidden_q.device)
    if ids is None:
        ids = torch.empty((T, top_k), dtype=torch.int32, device=hidden_q.device)
    args = (hidden_q.data_ptr(), hidden_scale.data_ptr(), gate_q.data_ptr(), gate_scale.data_ptr(), T, H, E,
            int(top_k), scores.data_ptr(), ids.data_ptr())
    fn, name = library().tk_gating_fused_topk_fp8, "tk_gating_fused_topk_fp8"
    if logits is not None and workspace is not None:
        raise ValueError("the FP8 workspace entry point has no logits variant")
    if logits is not None:
        _check_logits(logits, T, E, hidden_q.device)
        args = args + (logits.data_ptr(),)
        fn, name = library().tk_gating_fused_topk_fp8_logits, "tk_gating_fused_topk_fp8_logits"
    if workspace is not None:
        _check_workspace(workspace, hidden_q.device)
        args = args + (workspace.data_ptr(), workspace.numel() * workspace.element_size())
        fn, name = library().tk_gating_fused_topk_fp8_ws, "tk_gating_fused_topk_fp8_ws"
    with torch.cuda.device(hidden_q.device):
        st = fn(*args, _stream_handle(stream, hidden_q.device))
    _check(st, name)
    return scores, ids


def fused_topk_gating_host(hidden_host, gate_weight, top_k: int, scores_host, ids_host, hidden_dev, scores_dev,
                           ids_dev, stream=None) -> None:
    """End-to-end call: host ``hidden_host`` in, host ``scores_host``/``ids_host``
    out, through caller-owned device staging tensors; asynchronous on ``stream``."""
    T, H = hidden_host.shape
    E = gate_weight.shape[1]
    import torch
    with torch.cuda.device(gate_weight.device):
        st = library().tk_gating_fused_topk_host(
            hidden_host.data_ptr(), gate_weight.data_ptr(), T, H, E, int(top_k), scores_host.data_ptr(),
            ids_host.data_ptr(), hidden_dev.data_ptr(), scores_dev.data_ptr(), ids_dev.data_ptr(),
            _stream_handle(stream, gate_weight.device))
    _check(st, "tk_gating_fused_topk_host")


def make_plan(T: int, H: int, E: int, k: int, num_sms: int = 148) -> dict:
    """The launch the library would make (host logic only; no GPU needed)."""
    p = _Plan()
    st = library().tk_gating_make_plan(T, H, E, k, num_sms, ctypes.byref(p))
    _check(st, "tk_gating_make_plan")
    return {name: getattr(p, name) for name, _ in _Plan._fields_}


def device_error(clear: bool = True) -> int:
    """Device error word of the current device (0 = no kernel wait expired)."""
    w = ctypes.c_uint32(0)
    st = library().tk_gating_device_error(ctypes.byref(w), 1 if clear else 0)
    if st not in (TK_OK, TK_ERR_DEVICE_TIMEOUT):
        _check(st, "tk_gating_device_error")
    return int(w.value)


def clock_counters(clear: bool = True) -> dict:
    """SM-clock record of the gating launches on the current device since the
    last clear: ``{"sm_cycles", "elapsed_ns", "launches", "sm_ghz"}`` (first CTA
    of each launch, start to end; ``sm_ghz`` = cycles / ns, None without launches)."""
    c, n, l = ctypes.c_uint64(0), ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check(library().tk_gating_clock_counters(ctypes.byref(c), ctypes.byref(n), ctypes.byref(l), 1 if clear else 0),
           "tk_gating_clock_counters")
    return {"sm_cycles": int(c.value), "elapsed_ns": int(n.value), "launches": int(l.value),
            "sm_ghz": (c.value / n.value) if n.value else None}


def set_wait_timeout_ns(timeout_ns: int) -> None:
    _check(library().tk_gating_set_wait_timeout_ns(int(timeout_ns)), "tk_gating_set_wait_timeout_ns")


def route_plan(T: int, k: int, E: int, num_sms: int = 148) -> dict:
    """The launches ``route`` would make (host logic only; no GPU needed)."""
    p = _RoutePlan()
    _check(library().tk_gating_route_plan(T, k, E, num_sms, ctypes.byref(p)), "tk_gating_route_plan")
    return {name: getattr(p, name) for name, _ in _RoutePlan._fields_}


def route_ptr(ids: int, T: int, k: int, E: int, offsets: int, sorted_slots: int, slot_pos: int,
              stream: int = 0) -> int:
    """Raw C-ABI call with integer device pointers; returns the tk_status."""
    return int(library().tk_gating_route(ids, T, k, E, offsets, sorted_slots, slot_pos, stream))


def route(ids, num_experts: int, offsets=None, sorted_slots=None, slot_pos=None, stream=None):
    """Routing metadata of expert ids ``[T, k]`` (CUDA int32, contiguous):
    ``(offsets[E+1], sorted_slots[T*k], slot_pos[T,k])``, all int32 -- the
    assignments grouped by expert, ascending inside an expert.  Output tensors
    may be passed in.  The launches go on ``stream`` (default: the current
    torch stream)."""
    import torch
    if ids.dtype != torch.int32 or ids.dim() != 2 or not ids.is_cuda or not ids.is_contiguous():
        raise ValueError("ids must be a contiguous CUDA int32 [T, k] tensor")
    T, k = ids.shape
    E = int(num_experts)
    dev = ids.device
    if offsets is None:
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if sorted_slots is None:
        sorted_slots = torch.empty(T * k, dtype=torch.int32, device=dev)
    if slot_pos is None:
        slot_pos = torch.empty((T, k), dtype=torch.int32, device=dev)
    for name, t, n in (("offsets", offsets, E + 1), ("sorted_slots", sorted_slots, T * k),
                       ("slot_pos", slot_pos, T * k)):
        if t.dtype != torch.int32 or t.numel() != n or not t.is_contiguous() or t.device != dev:
            raise ValueError(f"{name} must be a contiguous int32 tensor of {n} elements on {dev}")
    with torch.cuda.device(dev):
        st = library().tk_gating_route(ids.data_ptr(), T, k, E, offsets.data_ptr(), sorted_slots.data_ptr(),
                                       slot_pos.data_ptr(), _stream_handle(stream, dev))
    _check(st, "tk_gating_route")
    return offsets, sorted_slots, slot_pos


def route_static_ptr(ids: int, T: int, k: int, E: int, offsets: int, sorted_slots: int, slot_pos: int,
                     stream: int = 0) -> int:
    """Raw C-ABI call of the no-allocation routing entry point (integer device
    pointers); returns the tk_status."""
    return int(library().tk_gating_route_static(ids, T, k, E, offsets, sorted_slots, slot_pos, stream))
