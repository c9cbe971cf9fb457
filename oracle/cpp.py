"""ctypes binding of the plain C++17 oracle (csa2_oracle.cpp), and a driver that
runs it over a synthetic workload's layer stack.

TEST INFRASTRUCTURE (see csa2_oracle.py): used only by the tests, smoke() and
the CPU-baseline and reference legs of the benchmark. The library is compiled
with g++ into this directory on first use.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, List, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.cpp")
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_handle = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, std::thread) if it is missing or stale."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-shared", "-fPIC", "-pthread", "-o", tmp, _SRC])
        os.replace(tmp, _SO)
    return _SO


def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def lib():
    global _handle
    with _lock:
        if _handle is None:
            L = ctypes.CDLL(build())
            i32, i64, vp, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
            L.orc_e2m1_value.argtypes = [i32]
            L.orc_e2m1_value.restype = dbl
            L.orc_e4m3_value.argtypes = [i32]
            L.orc_e4m3_value.restype = dbl
            L.orc_e2m1_round.argtypes = [dbl]
            L.orc_e2m1_round.restype = i32
            L.orc_e4m3_round.argtypes = [dbl]
            L.orc_e4m3_round.restype = i32
            L.orc_fp4_quantize.argtypes = [vp, i64, i32, vp, vp, i32]
            L.orc_compress_entries.argtypes = [vp, i64, i32, i32, vp]
            L.orc_compress_entries.restype = None
            L.orc_last_entry.argtypes = [i32, i32]
            L.orc_last_entry.restype = i32
            L.orc_fp4_value.argtypes = [vp, vp, i32]
            L.orc_fp4_value.restype = dbl
            L.orc_index_full.argtypes = [vp, vp, i32, i32, vp, i32, i32, i32, i32, vp, vp]
            L.orc_index_reindex.argtypes = [vp, vp, i32, i32, vp, vp, i32, i32, vp]
            L.orc_attention_unit.argtypes = [vp, i32, i32, vp, vp, vp, i32, vp, vp, i32, i32, i32, vp, vp]
            L.orc_index_full_batch.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, i64, i32, i32, vp, vp, i32]
            L.orc_index_reindex_batch.argtypes = [i32, i32, i32, i32, vp, vp, vp, i64, vp, i32, i32, vp, i32]
            L.orc_attention_batch.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32, vp, vp, i32, vp, i32,
                                              vp, vp, i32]
            for f in (L.orc_fp4_quantize, L.orc_index_full, L.orc_index_reindex, L.orc_attention_unit,
                      L.orc_index_full_batch, L.orc_index_reindex_batch, L.orc_attention_batch):
                f.restype = None
            _handle = L
    return _handle


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: Optional[np.ndarray]) -> Optional[int]:
    return None if a is None else a.ctypes.data


# ---------------------------------------------------------------- single units
def fp4_quantize(x: np.ndarray, threads: int = 0):
    x = _c(x, np.float32)
    D = x.shape[-1]
    rows = x.size // D
    codes = np.empty(x.shape[:-1] + (D // 2,), np.uint8)
    scales = np.empty(x.shape[:-1] + (D // 16,), np.uint8)
    lib().orc_fp4_quantize(_p(x), rows, D, _p(codes), _p(scales), threads or host_threads())
    return codes, scales


def compress_entries(x: np.ndarray, m: int) -> np.ndarray:
    """Entries of compression rate m from per-position rows [..., n, D]: [..., n / m, D]."""
    x = _c(x, np.float32)
    D = x.shape[-1]
    groups = x.size // D // m
    out = np.empty(x.shape[:-2] + (x.shape[-2] // m, D), np.float32)
    lib().orc_compress_entries(_p(x), groups, m, D, _p(out))
    return out


def last_entries(q_pos, m: int) -> np.ndarray:
    """The last global entry each query position may read."""
    q = np.asarray(q_pos, dtype=np.int32)
    L = lib()
    return np.vectorize(lambda t: L.orc_last_entry(int(t), m), otypes=[np.int32])(q) if q.size else q


def index_full(qi, w, keys, t: int, k: int, P: int = 0):
    qi, w, keys = _c(qi, np.int8), _c(w, np.int32), _c(keys, np.int8)
    Hi, Di = qi.shape
    topk = np.empty(k, np.int32)
    pool = np.empty(P, np.int32) if P > 0 else None
    lib().orc_index_full(_p(qi), _p(w), Hi, Di, _p(keys), keys.shape[0], t, k, P, _p(pool), _p(topk))
    return pool, topk


def index_reindex(qi, w, keys, pool_in, k: int):
    qi, w, keys, pool_in = _c(qi, np.int8), _c(w, np.int32), _c(keys, np.int8), _c(pool_in, np.int32)
    Hi, Di = qi.shape
    topk = np.empty(k, np.int32)
    lib().orc_index_reindex(_p(qi), _p(w), Hi, Di, _p(keys), _p(pool_in), pool_in.shape[0], k, _p(topk))
    return topk


def attention_unit(q_bits, codes_seq, scales_seq, topk, kl_bits, vl_bits, local_base: int, t: int, W: int):
    """q_bits [Hq, D] and kl_bits/vl_bits [Lloc, D] are bf16 bit patterns (uint16)."""
    q = _c(q_bits, np.uint16)
    Hq, D = q.shape
    codes_seq, scales_seq = _c(codes_seq, np.uint8), _c(scales_seq, np.uint8)
    topk = _c(topk, np.int32)
    kl = None if kl_bits is None else _c(kl_bits, np.uint16)
    vl = None if vl_bits is None else _c(vl_bits, np.uint16)
    out = np.empty((Hq, D), np.float64)
    lse = np.empty(Hq, np.float64)
    lib().orc_attention_unit(_p(q), Hq, D, _p(codes_seq), _p(scales_seq), _p(topk), topk.shape[0], _p(kl), _p(vl),
                             local_base, t, W, _p(out), _p(lse))
    return out, lse


# ---------------------------------------------------------------- batches (threads over units)
def index_full_batch(q_pos, qi, w, ki, k: int, P: int = 0, threads: int = 0):
    q_pos, qi, w, ki = _c(q_pos, np.int32), _c(qi, np.int8), _c(w, np.int32), _c(ki, np.int8)
    B, Tq, Hi, Di = qi.shape
    N = ki.shape[1]
    topk = np.empty((B, Tq, k), np.int32)
    pool = np.empty((B, Tq, P), np.int32) if P > 0 else None
    lib().orc_index_full_batch(B, Tq, N, Hi, Di, _p(q_pos), _p(qi), _p(w), _p(ki), N * Di, k, P, _p(pool), _p(topk),
                               threads or host_threads())
    return pool, topk


def index_reindex_batch(qi, w, ki, pool, k: int, threads: int = 0):
    qi, w, ki, pool = _c(qi, np.int8), _c(w, np.int32), _c(ki, np.int8), _c(pool, np.int32)
    B, Tq, Hi, Di = qi.shape
    topk = np.empty((B, Tq, k), np.int32)
    lib().orc_index_reindex_batch(B, Tq, Hi, Di, _p(qi), _p(w), _p(ki), ki.shape[1] * Di, _p(pool), pool.shape[-1], k,
                                  _p(topk), threads or host_threads())
    return topk


def attention_batch(q_pos, q_bits, codes, scales, topk, kl_bits, vl_bits, local_base, W: int, threads: int = 0):
    q_pos, q = _c(q_pos, np.int32), _c(q_bits, np.uint16)
    B, Tq, Hq, D = q.shape
    codes, scales, topk = _c(codes, np.uint8), _c(scales, np.uint8), _c(topk, np.int32)
    kl = None if (W == 0 or kl_bits is None) else _c(kl_bits, np.uint16)
    vl = None if (W == 0 or vl_bits is None) else _c(vl_bits, np.uint16)
    base = None if (W == 0 or local_base is None) else _c(local_base, np.int32)
    Lloc = 0 if kl is None else kl.shape[1]
    out = np.empty((B, Tq, Hq, D), np.float64)
    lse = np.empty((B, Tq, Hq), np.float64)
    lib().orc_attention_batch(B, Tq, codes.shape[1], Hq, D, _p(q_pos), _p(q), _p(codes), _p(scales), _p(topk),
                              topk.shape[-1], _p(kl), _p(vl), Lloc, _p(base), W, _p(out), _p(lse),
                              threads or host_threads())
    return out, lse


# ---------------------------------------------------------------- a workload's layer stack
class StackState:
    """What one layer hands to the next for a set of sequences of a synthetic
    workload: the current list and the most recent Full layer's pool ([CED] Fig. 5)."""

    def __init__(self, wl, seqs=None):
        self.wl = wl
        B = wl.spec.B
        self.seqs = list(range(B)) if seqs is None else list(seqs)
        self.all = self.seqs == list(range(B))
        self.cur = None
        self.pool = None

    def pick(self, a):
        return a if self.all else a[self.seqs]


def run_layer(st: StackState, li: int, codes=None, scales=None, threads: int = 0) -> Dict:
    """Layer li for every query of st's sequences: Full scores every causal position
    and keeps the pool and top-k; Reindex rescores the most recent Full pool; Reuse
    takes the current list. With codes/scales (the quantised cache of every
    sequence), also the layer's attention. Returns {mode, pool, topk[, out, lse]}."""
    wl = st.wl
    s = wl.spec
    L = s.layers[li]
    q_pos = st.pick(wl.q_pos())
    e = {"mode": L.mode, "pool": None}
    if L.mode == "FULL":
        q_ent = q_pos if s.m <= 1 else last_entries(q_pos, s.m)   # the bound on global entries
        p, st.cur = index_full_batch(q_ent, st.pick(wl.qi(li)), wl.w(li), st.pick(wl.ki(L.key_set)), L.k, L.P, threads)
        if p is not None:
            st.pool = p
        e["pool"] = p
    elif L.mode == "REINDEX":
        if st.pool is None:
            raise ValueError(f"layer {li}: REINDEX needs a pool from an earlier FULL layer")
        st.cur = index_reindex_batch(st.pick(wl.qi(li)), wl.w(li), st.pick(wl.ki(L.key_set)), st.pool, L.k, threads)
    elif st.cur is None:
        raise ValueError(f"layer {li}: REUSE needs an earlier FULL or REINDEX layer")
    e["topk"] = st.cur
    if codes is not None:
        e["out"], e["lse"] = attention_batch(q_pos, st.pick(wl.q(li)), st.pick(codes), st.pick(scales), st.cur,
                                             st.pick(wl.kl(li)), st.pick(wl.vl(li)), st.pick(wl.local_base_arr()),
                                             s.W, threads)
    return e


def stack_lists(wl, threads: int = 0) -> List[Dict]:
    """Index lists of every query of a synthetic workload through its layer stack:
    per layer {mode, pool, topk} as [B, Tq, ...] arrays."""
    st = StackState(wl)
    return [run_layer(st, li, threads=threads) for li in range(wl.spec.L)]


def stack_outputs(wl, codes, scales, lists: List[Dict], seqs, threads: int = 0) -> List[Dict]:
    """Attention outputs of the given sequences' queries at every layer, from the
    layer lists of stack_lists: per layer {out [len(seqs), Tq, Hq, D], lse}."""
    s = wl.spec
    seqs = list(seqs)
    q_pos = wl.q_pos()[seqs]
    base = wl.local_base_arr()[seqs]
    out = []
    for li in range(s.L):
        o, l = attention_batch(q_pos, wl.q(li)[seqs], codes[seqs], scales[seqs], lists[li]["topk"][seqs],
                               wl.kl(li)[seqs], wl.vl(li)[seqs], base, s.W, threads)
        out.append({"out": o, "lse": l})
    return out
