"""Seeded synthetic router workloads (inputs only).

The gating pages (chenxutan.com "TileKernels 深度解析", section 4.1 "MoE Gating")
give the operator but no data, so every input here is synthetic: hidden states
``x[T, H]`` and a gate matrix ``w[H, E]``, both bf16, drawn from a counter-based
normal generator (``synth.c``).  This module holds no gating arithmetic; the
oracle and the CUDA path both take their inputs from here.

Workloads (shapes follow the DeepSeek-style router the pages use: 256 experts,
hidden size 7168, top-8):

* ``tiny``      T=64,    H=512,  E=16,  k=2
* ``deepseek``  T=4096,  H=7168, E=256, k=8
* ``skew``      T=16384, H=4096, E=64,  k=6, with a shared direction ``u`` added
  to every token, four dominant experts whose gate columns equal ``u`` and four
  pairs of duplicated gate columns (exact ties)
* ``train``     T=65536, H=7168, E=256, k=8
* ``decode_T{1,8,32,128,256}``  H=7168, E=256, k=8

Arrays are returned as numpy ``uint16`` holding bf16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

STREAM_HIDDEN = 1
STREAM_GATE = 2
STREAM_UNIT = 3

# skew workload structure (our choice; the pages fix no indices)
SKEW_DOMINANT = (5, 17, 33, 60)
SKEW_DUPLICATE_PAIRS = ((10, 11), (20, 21), (40, 41), (62, 63))
SKEW_ALPHA = 3.0

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``libsynth.so`` (gcc, OpenMP) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i64, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
            vp = ctypes.c_void_p
            lib.synth_normal_f64.argtypes = [u64, u64, i64, i64, vp]
            lib.synth_normal_bf16.argtypes = [u64, u64, i64, i64, dbl, vp]
            lib.synth_normal_plus_vec_bf16.argtypes = [u64, u64, i64, i64, i64, vp, dbl, vp]
            lib.synth_round_bf16.argtypes = [vp, i64, vp]
            for f in (lib.synth_normal_f64, lib.synth_normal_bf16,
                      lib.synth_normal_plus_vec_bf16, lib.synth_round_bf16):
                f.restype = None
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def normal_f64(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.float64)
    if count:
        _load().synth_normal_f64(seed, stream, start, count, _ptr(out))
    return out


def normal_bf16(seed: int, stream: int, start: int, count: int, scale: float = 1.0) -> np.ndarray:
    out = np.empty(count, dtype=np.uint16)
    if count:
        _load().synth_normal_bf16(seed, stream, start, count, float(scale), _ptr(out))
    return out


def round_bf16(values: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    if v.size:
        _load().synth_round_bf16(_ptr(v), v.size, _ptr(out))
    return out


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@dataclass(frozen=True)
class RouterWorkload:
    name: str
    T: int
    H: int
    E: int
    k: int
    kind: str = "normal"  # "normal" | "skew"
    seed: int = 0
    dominant: tuple = field(default=())
    duplicate_pairs: tuple = field(default=())

    # -- generation -------------------------------------------------------
    def unit_vector(self) -> np.ndarray:
        u = normal_f64(self.seed, STREAM_UNIT, 0, self.H)
        return u / np.sqrt(np.dot(u, u))

    def gate_weight(self) -> np.ndarray:
        """``w[H, E]`` bf16 bits, row-major; ~N(0, 1/H) plus the skew structure."""
        w = normal_bf16(self.seed, STREAM_GATE, 0, self.H * self.E, 1.0 / np.sqrt(self.H))
        w = w.reshape(self.H, self.E)
        if self.kind == "skew":
            ub = round_bf16(self.unit_vector())
            for d in self.dominant:
                w[:, d] = ub
            for a, b in self.duplicate_pairs:
                w[:, b] = w[:, a]
        return w

    def hidden_rows(self, row0: int, nrows: int) -> np.ndarray:
        """Rows ``[row0, row0 + nrows)`` of ``x[T, H]`` bf16 bits."""
        assert 0 <= row0 and row0 + nrows <= self.T
        if self.kind == "skew":
            out = np.empty((nrows, self.H), dtype=np.uint16)
            if nrows:
                u = np.ascontiguousarray(self.unit_vector())
                _load().synth_normal_plus_vec_bf16(self.seed, STREAM_HIDDEN, row0, nrows, self.H,
                                                   _ptr(u), SKEW_ALPHA, _ptr(out))
            return out
        return normal_bf16(self.seed, STREAM_HIDDEN, row0 * self.H, nrows * self.H).reshape(nrows, self.H)

    def hidden(self) -> np.ndarray:
        return self.hidden_rows(0, self.T)

    def with_T(self, T: int) -> "RouterWorkload":
        return RouterWorkload(self.name, T, self.H, self.E, self.k, self.kind, self.seed,
                              self.dominant, self.duplicate_pairs)

    # -- algorithmic work (per call) ---------------------------------------
    def algorithmic_bytes(self) -> int:
        """hidden read once + gate read once + scores/ids written once."""
        return 2 * self.T * self.H + 2 * self.H * self.E + 8 * self.T * self.k

    def flops(self) -> int:
        return 2 * self.T * self.H * self.E


TINY = RouterWorkload("tiny", 64, 512, 16, 2)
DEEPSEEK = RouterWorkload("deepseek", 4096, 7168, 256, 8)
SKEW = RouterWorkload("skew", 16384, 4096, 64, 6, kind="skew",
                      dominant=SKEW_DOMINANT, duplicate_pairs=SKEW_DUPLICATE_PAIRS)
TRAIN = RouterWorkload("train", 65536, 7168, 256, 8)
DECODE_TS = (1, 8, 32, 128, 256)
DECODE = tuple(RouterWorkload(f"decode_T{t}", t, 7168, 256, 8) for t in DECODE_TS)

# More experts and larger k than the pages' router (fine-grained MoE): two MMA
# chunks of 256 experts, top-32 selection.
LARGE_E = RouterWorkload("large_e", 65536, 7168, 512, 8)
LARGE_K = RouterWorkload("large_k", 4096, 7168, 512, 32)
E1024 = RouterWorkload("e1024", 65536, 7168, 1024, 8)  # two expert groups of 512

WORKLOADS = {w.name: w for w in (TINY, DEEPSEEK, SKEW, TRAIN, LARGE_E, LARGE_K, E1024) + DECODE}


def quantize_e4m3_rows(values: np.ndarray):
    """Per-row FP8 E4M3 quantization of a float array [R, C]: scale = max|row| / 448
    (1 for an all-zero row), bits = e4m3(row / scale) rounded to nearest even by
    torch's float8_e4m3fn cast.  Returns (uint8 bits [R, C], float32 scales [R]).
    Input preparation only (the pages' per-token quantize); no gating arithmetic."""
    import torch
    v = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32))
    amax = v.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (v / scale[:, None]).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).numpy().copy(), scale.numpy().astype(np.float32)


def fp8_inputs(wl: "RouterWorkload"):
    """FP8 versions of a workload's inputs: the bf16 hidden rows quantized per token,
    the bf16 gate quantized per expert and stored expert-major [E, H].
    Returns (hidden_q [T, H], hidden_scale [T], gate_q [E, H], gate_scale [E])."""
    def to_f32(bits):  # exact bf16 -> fp32 widening
        return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    xq, xs = quantize_e4m3_rows(to_f32(wl.hidden()))
    wq, ws = quantize_e4m3_rows(np.ascontiguousarray(to_f32(wl.gate_weight()).T))
    return xq, xs, wq, ws


def expert_ids(T: int, k: int, E: int, seed: int, kind: str = "uniform") -> np.ndarray:
    """Seeded int32 ``[T, k]`` expert ids, k distinct per row (as a router emits).

    ``uniform``: every expert equally likely.  ``skew``: expert popularity drawn
    from a Dirichlet(0.3) (a few hot experts, a long cold tail), rows sampled
    without replacement by the Gumbel-top-k rule.  Inputs for the routing
    metadata only; nothing of the routing itself is computed here.
    """
    if not 1 <= k <= E:
        raise ValueError(f"need 1 <= k <= E, got k={k} E={E}")
    rng = np.random.default_rng(seed)
    keys = rng.random((T, E), dtype=np.float32)
    if kind == "skew":
        logp = np.log(rng.dirichlet(np.full(E, 0.3)) + 1e-30).astype(np.float32)
        keys = logp[None, :] - np.log(-np.log(np.maximum(keys, np.float32(1e-12))))
    elif kind != "uniform":
        raise ValueError(f"unknown kind {kind!r}")
    return np.argpartition(-keys, k - 1, axis=1)[:, :k].astype(np.int32) if T else np.zeros((0, k), np.int32)


def to_torch_bf16(bits: np.ndarray):
    """View a uint16 bf16-bit array as a CPU ``torch.bfloat16`` tensor (no copy)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
