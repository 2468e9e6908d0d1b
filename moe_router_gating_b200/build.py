"""Build the in-tree CUDA library ``libtk_gating.so`` for sm_100a with nvcc.

Usage: ``python -m moe_router_gating_b200.build [--verbose] [--debug]``
(``--verbose`` prints ptxas register / shared-memory usage; ``--debug`` builds
``libtk_gating_debug.so`` with the kernels' index checks compiled in).  Rebuilds only when a source or
the public header is newer than the library.
"""
from __future__ import annotations

import glob
import hashlib
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtk_gating.so")
# the same library with the kernels' index checks compiled in (TK_GATING_DEBUG)
DEBUG_LIB = os.path.join(PKG, "libtk_gating_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]
LINK_FLAGS = ["-shared", "-cudart", "static", "-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


# Sources that compile into the fused gating kernels (not the routing kernels).
GATING_KERNEL_SOURCES = ("tk_gating.cu", "gating_launch.cuh", "gating_launch_impl.cuh", "gating_bf16.cu",
                         "gating_fp8.cu", "gating_row_tiles.cuh", "gating_split_h.cuh", "gating_few_tokens.cuh",
                         "sm100_ptx.cuh", "route_counts.cuh", "topk_epilogue.cuh", "topk_merge.cuh")


def _code_only(text: str) -> str:
    """Source text without comments and blank lines (string literals here hold no comment markers)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def gating_kernel_digest() -> str:
    """Digest of the gating kernels' code (comments ignored): a profile measured on
    these kernels stays valid while it is unchanged."""
    h = hashlib.sha256()
    for name in GATING_KERNEL_SOURCES:
        with open(os.path.join(CSRC, name)) as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every csrc/*.cu to an object in parallel (the bf16 and FP8 kernel
    instances live in separate translation units), then link the library.
    ``debug`` builds libtk_gating_debug.so, with the kernels' index checks
    (TK_GATING_DEBUG: a failed check sets a bit of the device error word and
    skips the access)."""
    target = DEBUG_LIB if debug else LIB
    if not force and not is_stale(target):
        return target
    objdir = os.path.join(PKG, f"_build_{'debug_' if debug else ''}{os.getpid()}")
    os.makedirs(objdir, exist_ok=True)
    try:
        procs = []
        for src in sources():
            obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
            cmd = [nvcc(), *NVCC_FLAGS, *(["-DTK_GATING_DEBUG"] if debug else []), "-I", INCLUDE, "-I", CSRC, "-c",
                   src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            procs.append((src, obj, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
        failed = []
        for src, _, proc in procs:
            out, _ = proc.communicate()
            if out:
                sys.stdout.write(out)
            if proc.returncode != 0:
                failed.append(os.path.basename(src))
        if failed:
            raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(failed)})")
        tmp = target + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc(), *LINK_FLAGS, *[obj for _, obj, _ in procs], "-o", tmp])
        os.replace(tmp, target)
    finally:
        shutil.rmtree(objdir, ignore_errors=True)
    return target


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
