"""Build the CSA2 CUDA library (libcsa2.so) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libcsa2.so")
SOURCES = ["csa2_api.cu", "indexer.cu", "attention.cu", "fp4_quant.cu", "cache_append.cu"]
HEADERS = ["csa2_common.cuh", "fp4_codec.cuh", os.path.join("..", "..", "include", "csa2.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    deps = [src] + [os.path.join(CSRC, h) for h in HEADERS]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


LIB_CHECKED = os.path.join(HERE, "libcsa2_checked.so")
LIB_TRACE = os.path.join(HERE, "libcsa2_trace.so")


def build(force: bool = False, verbose: bool = False, extra=None, checked: bool = False, trace: bool = False) -> str:
    """Build libcsa2.so; with checked=True the range-checked libcsa2_checked.so
    (-DCSA2_CHECKED: computed indices are checked and reported instead of accessed); with
    trace=True the phase-trace libcsa2_trace.so (-DCSA2_PHASE_TRACE: kernels record phase clocks
    and per-CTA start and end times into host-registered buffers)."""
    lib = LIB_CHECKED if checked else LIB_TRACE if trace else LIB
    extra = list(extra or []) + (["-DCSA2_CHECKED"] if checked else []) + (["-DCSA2_PHASE_TRACE"] if trace else [])
    objdir = os.path.join(HERE, "_build_checked" if checked else "_build_trace" if trace else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs, changed = [], False
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(objdir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, s):
            cmd = [NVCC, *FLAGS, *extra, "-c", s, "-o", o]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)
            changed = True
    if changed or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *objs, "-lcudart"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, checked="--checked" in sys.argv, trace="--trace" in sys.argv)
