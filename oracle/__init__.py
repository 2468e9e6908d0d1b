"""CPU oracle for fused MoE top-k gating -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (``moe_router_gating_b200``)
never does, and this package imports nothing from the product.

The arithmetic lives in ``gating_oracle.c`` (plain C, fp64, full per-row sort),
written from the naive three-step form on the chenxutan.com page, section 4.1
"MoE Gating": logits = hidden @ gate_weight; top-k of the logits; softmax of
the k selected values; and in ``route_oracle.c`` (a stable counting sort of the
token-expert assignments, section 4.2 "MoE Routing"), and in
``gating_fp8_oracle.c`` (the same gating on FP8 E4M3 inputs with per-token and
per-expert scales, section 4.3 "Quantization").  Every function is pinned by
``tests/test_oracle_pins.py`` / ``tests/test_route_oracle.py`` /
``tests/test_fp8_oracle.py``; no part is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "gating_oracle.c")
ROUTE_SOURCE = os.path.join(_HERE, "route_oracle.c")
FP8_SOURCE = os.path.join(_HERE, "gating_fp8_oracle.c")
_LIB = os.path.join(_HERE, "libgating_oracle.so")
GCC_FLAGS = ["-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off"]

_lock = threading.Lock()
_libs: dict = {}


def compile_oracle(src: str, out: str, route_src: str = ROUTE_SOURCE, fp8_src: str = FP8_SOURCE) -> str:
    """Compile a gating-oracle source (possibly a modified copy) with the routing and FP8 oracles."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *GCC_FLAGS, src, route_src, fp8_src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    stale = not os.path.exists(_LIB) or any(os.path.getmtime(_LIB) < os.path.getmtime(f)
                                            for f in (SOURCE, ROUTE_SOURCE, FP8_SOURCE))
    if force or stale:
        compile_oracle(SOURCE, _LIB)
    return _LIB


@dataclass
class RouteResult:
    offsets: np.ndarray       # int32 [E + 1]
    sorted_slots: np.ndarray  # int32 [n]
    slot_pos: np.ndarray      # int32 [n]


@dataclass
class OracleResult:
    scores: np.ndarray    # fp32 [T, k]
    scores64: np.ndarray  # fp64 [T, k]
    ids: np.ndarray       # int32 [T, k]
    gap: np.ndarray       # fp64 [T]
    logits: np.ndarray | None  # fp64 [T, E] when requested


class Oracle:
    """ctypes handle on one compiled copy of the oracle source."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        lib.oracle_fused_topk_gating.argtypes = [vp, vp, i64, i64, i64, ctypes.c_int, vp, vp, vp, vp, vp]
        lib.oracle_fused_topk_gating.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_fused_topk_gating_fp8.argtypes = [vp, vp, vp, vp, i64, i64, i64, ctypes.c_int, vp, vp, vp, vp, vp]
        lib.oracle_fused_topk_gating_fp8.restype = ctypes.c_int
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_route.argtypes = [vp, i64, ctypes.c_int32, vp, vp, vp]
        lib.oracle_route.restype = ctypes.c_int
        self._lib = lib

    def max_threads(self) -> int:
        return int(self._lib.oracle_max_threads())

    def gating(self, hidden_bits: np.ndarray, gate_bits: np.ndarray, k: int,
               want_logits: bool = False) -> OracleResult:
        x = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
        w = np.ascontiguousarray(gate_bits, dtype=np.uint16)
        T, H = x.shape
        H2, E = w.shape
        if H != H2:
            raise ValueError(f"hidden is [T,{H}] but gate_weight is [{H2},E]")
        scores = np.zeros((T, k), dtype=np.float32)
        scores64 = np.zeros((T, k), dtype=np.float64)
        ids = np.full((T, k), -1, dtype=np.int32)
        gap = np.zeros(T, dtype=np.float64)
        logits = np.zeros((T, E), dtype=np.float64) if want_logits else None
        rc = self._lib.oracle_fused_topk_gating(
            x.ctypes.data, w.ctypes.data, T, H, E, k, scores.ctypes.data, scores64.ctypes.data,
            ids.ctypes.data, gap.ctypes.data, logits.ctypes.data if logits is not None else None)
        if rc != 0:
            raise ValueError(f"oracle_fused_topk_gating returned {rc} (T={T} H={H} E={E} k={k})")
        return OracleResult(scores, scores64, ids, gap, logits)


    def e4m3_to_f64(self, bits: int) -> float:
        return float(self._lib.oracle_e4m3_to_f64(int(bits) & 0xFF))

    def gating_fp8(self, hidden_q: np.ndarray, hidden_scale: np.ndarray, gate_q: np.ndarray,
                   gate_scale: np.ndarray, k: int, want_logits: bool = False) -> OracleResult:
        """``hidden_q`` e4m3 bits [T, H] with ``hidden_scale`` [T]; ``gate_q`` e4m3 bits
        [E, H] (expert-major) with ``gate_scale`` [E]."""
        xq = np.ascontiguousarray(hidden_q, dtype=np.uint8)
        wq = np.ascontiguousarray(gate_q, dtype=np.uint8)
        xs = np.ascontiguousarray(hidden_scale, dtype=np.float32)
        ws = np.ascontiguousarray(gate_scale, dtype=np.float32)
        T, H = xq.shape
        E, H2 = wq.shape
        if H != H2 or xs.shape != (T,) or ws.shape != (E,):
            raise ValueError("shapes do not chain: hidden_q [T,H], hidden_scale [T], gate_q [E,H], gate_scale [E]")
        scores = np.zeros((T, k), dtype=np.float32)
        scores64 = np.zeros((T, k), dtype=np.float64)
        ids = np.full((T, k), -1, dtype=np.int32)
        gap = np.zeros(T, dtype=np.float64)
        logits = np.zeros((T, E), dtype=np.float64) if want_logits else None
        rc = self._lib.oracle_fused_topk_gating_fp8(
            xq.ctypes.data, xs.ctypes.data, wq.ctypes.data, ws.ctypes.data, T, H, E, k, scores.ctypes.data,
            scores64.ctypes.data, ids.ctypes.data, gap.ctypes.data, logits.ctypes.data if logits is not None else None)
        if rc != 0:
            raise ValueError(f"oracle_fused_topk_gating_fp8 returned {rc} (T={T} H={H} E={E} k={k})")
        return OracleResult(scores, scores64, ids, gap, logits)

    def route(self, ids: np.ndarray, E: int) -> RouteResult:
        flat = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
        n = flat.size
        offsets = np.zeros(E + 1, dtype=np.int32)
        sorted_slots = np.full(n, -1, dtype=np.int32)
        slot_pos = np.full(n, -1, dtype=np.int32)
        rc = self._lib.oracle_route(flat.ctypes.data, n, E, offsets.ctypes.data, sorted_slots.ctypes.data,
                                    slot_pos.ctypes.data)
        if rc != 0:
            raise ValueError(f"oracle_route returned {rc} (n={n} E={E})")
        return RouteResult(offsets, sorted_slots, slot_pos)


def load(lib_path: str | None = None) -> Oracle:
    path = lib_path or build()
    with _lock:
        if path not in _libs:
            _libs[path] = Oracle(path)
        return _libs[path]


def fused_topk_gating(hidden_bits: np.ndarray, gate_bits: np.ndarray, k: int,
                      want_logits: bool = False) -> OracleResult:
    """Oracle result for bf16-bit inputs ``hidden[T,H]`` and ``gate_weight[H,E]``."""
    return load().gating(hidden_bits, gate_bits, k, want_logits)


def fused_topk_gating_fp8(hidden_q, hidden_scale, gate_q, gate_scale, k: int,
                          want_logits: bool = False) -> OracleResult:
    """Oracle result for FP8 (E4M3) inputs with per-token and per-expert scales."""
    return load().gating_fp8(hidden_q, hidden_scale, gate_q, gate_scale, k, want_logits)


def route(ids: np.ndarray, E: int) -> RouteResult:
    """Oracle routing metadata for expert ids ``[T, k]`` (or flat ``[T*k]``)."""
    return load().route(ids, E)
