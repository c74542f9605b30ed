"""Builds the in-tree CUDA library libgqe.so for sm_100a (B200).

Usage:  python moe_gqa_query_b200/build.py   (or build_library() from Python)
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libgqe.so")
# diagnostic build: the same sources with the attention kernel's CTA timeline
# recorded (include/gqe_trace.h)
TRACE_LIB = os.path.join(PKG, "libgqe_trace.so")
TRACE_FLAGS = ["-DGQE_ATTN_TRACE"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-warn-spills",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def build_library(verbose: bool = False, extra=(), trace: bool = False) -> str:
    """Compile every CUDA source into moe_gqa_query_b200/libgqe.so (or, with
    trace=True, the diagnostic libgqe_trace.so)."""
    out = TRACE_LIB if trace else LIB
    extra = tuple(extra) + (tuple(TRACE_FLAGS) if trace else ())
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    if os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in deps) and not extra:
        return out
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-o", out + ".tmp", *sources()]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libgqe.so")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    args = sys.argv[1:]
    trace = "--trace" in args
    print(build_library(verbose=True, extra=tuple(a for a in args if a != "--trace"), trace=trace))
