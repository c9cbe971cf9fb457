"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This package only draws random numbers (see ``gen.c`` for the generator's
definition) and lays them out in the shapes of the workloads. It contains none
of the method's arithmetic: no scoring, selection, quantisation or attention.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_SO = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_handle = None


def build(force: bool = False) -> str:
    """Compile the generator with gcc (OpenMP threads) if it is missing or stale."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _lib():
    global _handle
    with _lock:
        if _handle is None:
            lib = ctypes.CDLL(build())
            u64, i64, i32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
            lib.synth_randint_i8.argtypes = [u64, u64, i64, i64, i32, i32, vp]
            lib.synth_randint_i32.argtypes = [u64, u64, i64, i64, i32, i32, vp]
            lib.synth_normal_f32.argtypes = [u64, u64, i64, i64, vp]
            lib.synth_normal_bf16.argtypes = [u64, u64, i64, i64, vp]
            _handle = lib
    return _handle


def _count(shape) -> int:
    return int(np.prod(shape, dtype=np.int64)) if len(shape) else 1


def randint_i8(seed: int, tid: int, shape, lo: int = -127, hi: int = 127, start: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=np.int8)
    _lib().synth_randint_i8(seed, tid, start, _count(shape), lo, hi, out.ctypes.data)
    return out


def randint_i32(seed: int, tid: int, shape, lo: int, hi: int, start: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=np.int32)
    _lib().synth_randint_i32(seed, tid, start, _count(shape), lo, hi, out.ctypes.data)
    return out


def normal_f32(seed: int, tid: int, shape, start: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _lib().synth_normal_f32(seed, tid, start, _count(shape), out.ctypes.data)
    return out


def normal_bf16(seed: int, tid: int, shape, start: int = 0) -> np.ndarray:
    """Standard normals as bf16 bit patterns (uint16)."""
    out = np.empty(shape, dtype=np.uint16)
    _lib().synth_normal_bf16(seed, tid, start, _count(shape), out.ctypes.data)
    return out


from .workloads import CONFIGS, Workload, make_workload  # noqa: E402,F401
