"""Build libpod_attn.so in-tree with nvcc for sm_100a.

Usage: ``python -m hybrid_prefill_decode_pod_b200.build [--force]``.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpod_attn.so")
SOURCES = [os.path.join(CSRC, "pod_kernels.cu"), os.path.join(CSRC, "pod_attn_api.cpp"),
           os.path.join(CSRC, "pod_static.cu")]
HEADERS = [os.path.join(CSRC, f) for f in ("pod_plan.h", "pod_ptx.cuh", "pod_exp2.cuh", "pod_prefill.cuh")] + [
    os.path.join(INCLUDE, "pod_attn.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-I", INCLUDE, "-I", CSRC,
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile the library. POD_ATTN_NVCC_EXTRA (space-separated) adds flags,
    e.g. -DPOD_SOFT_EXP2_PAIRS=4, for tuning builds."""
    extra = list(extra) + os.environ.get("POD_ATTN_NVCC_EXTRA", "").split()
    if not force and not _stale() and not os.environ.get("POD_ATTN_NVCC_EXTRA"):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-shared", "-o", tmp, *SOURCES, "-lcudart"]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
    print(LIB)
