"""ctypes view of the C ABI in include/csa2.h (argument marshalling only).

The functions here carry the same names as the C entry points and take the
same structures; every step of the computation runs in libcsa2.so. Loading
fails loudly when the library cannot be built or loaded.
"""
from __future__ import annotations

import ctypes
import os
import threading
from ctypes import POINTER, Structure, c_char_p, c_int, c_int32, c_int64, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
_lock = threading.Lock()
_lib = None

CSA2_FULL, CSA2_REINDEX, CSA2_REUSE = 0, 1, 2
MODES = {"FULL": CSA2_FULL, "REINDEX": CSA2_REINDEX, "REUSE": CSA2_REUSE}

STATUS_NAMES = {
    0: "CSA2_OK", 1: "CSA2_ERR_NULL", 2: "CSA2_ERR_SHAPE", 3: "CSA2_ERR_ALIGN", 4: "CSA2_ERR_MODE",
    5: "CSA2_ERR_RANGE", 6: "CSA2_ERR_UNSUPPORTED", 7: "CSA2_ERR_CUDA", 8: "CSA2_ERR_TIMEOUT",
    9: "CSA2_ERR_WORKSPACE",
}


class IndexArgs(Structure):
    _fields_ = [
        ("B", c_int32), ("Tq", c_int32), ("N", c_int32), ("Hi", c_int32), ("Di", c_int32),
        ("k", c_int32), ("P", c_int32), ("mode", c_int32),
        ("q_pos", c_void_p), ("qi", c_void_p), ("w", c_void_p), ("ki", c_void_p),
        ("ki_seq_stride", c_int64), ("pool_in", c_void_p), ("P_in", c_int32),
        ("pool_out", c_void_p), ("topk_out", c_void_p), ("m", c_int32),
    ]


class AttnArgs(Structure):
    _fields_ = [
        ("B", c_int32), ("Tq", c_int32), ("N", c_int32), ("Hq", c_int32), ("D", c_int32),
        ("k", c_int32), ("W", c_int32), ("Lloc", c_int32),
        ("q_pos", c_void_p), ("q", c_void_p), ("kv_fp4", c_void_p), ("kv_scale", c_void_p),
        ("topk", c_void_p), ("kl", c_void_p), ("vl", c_void_p), ("local_base", c_void_p),
        ("out", c_void_p), ("lse", c_void_p), ("m", c_int32),
    ]


class AppendArgs(Structure):
    _fields_ = [
        ("B", c_int32), ("N", c_int32), ("D", c_int32), ("Di", c_int32), ("S", c_int32), ("L", c_int32),
        ("W", c_int32), ("Lcap", c_int32),
        ("pos", c_void_p), ("kv_new", c_void_p), ("kv_fp4", c_void_p), ("kv_scale", c_void_p),
        ("ki_new", c_void_p), ("ki", c_void_p), ("kl_new", c_void_p), ("vl_new", c_void_p),
        ("kl", c_void_p), ("vl", c_void_p), ("local_base", c_void_p),
    ]


class StackArgs(Structure):
    _fields_ = [("L", c_int32), ("idx", POINTER(IndexArgs)), ("attn", POINTER(AttnArgs))]


EXPORTED = ("csa2_workspace_bytes", "csa2_index_topk", "csa2_sparse_attn", "csa2_layer_stack",
            "csa2_fp4_quantize", "csa2_status_string", "csa2_set_wait_controls", "csa2_sparse_attn_noalloc", "csa2_cache_append",
            "csa2_fp4_compress")


def checked_library() -> bool:
    """CSA2_LIBRARY=checked selects the range-checked build (libcsa2_checked.so)."""
    return os.environ.get("CSA2_LIBRARY", "") == "checked"


def trace_library() -> bool:
    """CSA2_LIBRARY=trace selects the phase-trace build (libcsa2_trace.so)."""
    return os.environ.get("CSA2_LIBRARY", "") == "trace"


def library_path() -> str:
    name = "libcsa2_checked.so" if checked_library() else "libcsa2_trace.so" if trace_library() else "libcsa2.so"
    return os.path.join(_HERE, name)


def lib():
    """Load libcsa2.so (building it first if it is missing or older than its sources)."""
    global _lib
    with _lock:
        if _lib is None:
            from . import build as _build
            try:
                path = _build.build(checked=checked_library(), trace=trace_library())
            except Exception as e:  # noqa: BLE001
                raise RuntimeError(f"cannot build the CSA2 CUDA library: {e}") from e
            L = ctypes.CDLL(path)
            L.csa2_workspace_bytes.argtypes = [c_int, c_void_p]
            L.csa2_workspace_bytes.restype = c_size_t
            for name, st in (("csa2_index_topk", IndexArgs), ("csa2_sparse_attn", AttnArgs),
                             ("csa2_layer_stack", StackArgs)):
                f = getattr(L, name)
                f.argtypes = [POINTER(st), c_void_p, c_size_t, c_void_p, c_void_p]
                f.restype = c_int
            L.csa2_fp4_quantize.argtypes = [c_void_p, c_int64, c_int32, c_void_p, c_void_p, c_void_p]
            L.csa2_fp4_quantize.restype = c_int
            L.csa2_fp4_compress.argtypes = [c_void_p, c_int64, c_int32, c_int32, c_void_p, c_void_p, c_void_p]
            L.csa2_fp4_compress.restype = c_int
            L.csa2_cache_append.argtypes = [POINTER(AppendArgs), c_void_p, c_void_p]
            L.csa2_cache_append.restype = c_int
            L.csa2_set_wait_controls.argtypes = [c_int64, c_int32]
            L.csa2_set_wait_controls.restype = c_int
            L.csa2_status_string.argtypes = [c_int]
            L.csa2_status_string.restype = c_char_p
            if trace_library():   # (slots, rows, on, timeline, counter, capacity)
                for name in ("csa2_trace_set_idx", "csa2_trace_set_attn"):
                    f = getattr(L, name)
                    f.argtypes = [c_void_p, ctypes.c_uint, c_int, c_void_p, c_void_p, ctypes.c_uint]
                    f.restype = c_int
            _lib = L
    return _lib


def csa2_workspace_bytes(which: int, args) -> int:
    return lib().csa2_workspace_bytes(which, ctypes.cast(ctypes.pointer(args), c_void_p))


def csa2_index_topk(args: IndexArgs, workspace: int, ws_bytes: int, d_status: int, stream: int) -> int:
    return lib().csa2_index_topk(ctypes.byref(args), workspace, ws_bytes, d_status, stream)


def csa2_sparse_attn(args: AttnArgs, workspace: int, ws_bytes: int, d_status: int, stream: int) -> int:
    return lib().csa2_sparse_attn(ctypes.byref(args), workspace, ws_bytes, d_status, stream)


def csa2_layer_stack(args: StackArgs, workspace: int, ws_bytes: int, d_status: int, stream: int) -> int:
    return lib().csa2_layer_stack(ctypes.byref(args), workspace, ws_bytes, d_status, stream)


def csa2_fp4_quantize(x: int, rows: int, D: int, fp4: int, scale: int, stream: int) -> int:
    return lib().csa2_fp4_quantize(x, rows, D, fp4, scale, stream)


def csa2_cache_append(args: AppendArgs, d_status: int, stream: int) -> int:
    return lib().csa2_cache_append(ctypes.byref(args), d_status, stream)


def csa2_set_wait_controls(budget_cycles: int, skip_arrival: int) -> int:
    return lib().csa2_set_wait_controls(budget_cycles, skip_arrival)


def csa2_fp4_compress(x: int, groups: int, m: int, D: int, fp4: int, scale: int, stream: int) -> int:
    return lib().csa2_fp4_compress(x, groups, m, D, fp4, scale, stream)


def csa2_status_string(code: int) -> str:
    return lib().csa2_status_string(code).decode()


class Csa2Error(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        name = STATUS_NAMES.get(code, str(code))
        msg = f"{where}: {name}" if where else name
        try:
            msg += f" ({csa2_status_string(code)})"
        except Exception:  # noqa: BLE001
            pass
        super().__init__(msg)


def check(code: int, where: str = "") -> None:
    if code != 0:
        raise Csa2Error(code, where)
