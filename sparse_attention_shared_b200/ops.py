"""PyTorch-facing wrappers over the C ABI: device memory, streams and argument
marshalling only. Every step of the computation runs in libcsa2.so."""
from __future__ import annotations

import ctypes
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

from . import capi
from .capi import AttnArgs, IndexArgs, StackArgs, check


def _ptr(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    return int((stream or torch.cuda.current_stream()).cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("CSA2 ops take CUDA tensors")


class Workspace:
    """Caller-owned device workspace, zero-filled when (re)allocated."""

    def __init__(self, device: str = "cuda"):
        self.device = device
        self.buf: Optional[torch.Tensor] = None

    def get(self, nbytes: int) -> torch.Tensor:
        if nbytes <= 0:
            raise ValueError("invalid arguments (workspace size query returned 0)")
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf

    def reset(self) -> None:
        if self.buf is not None:
            self.buf.zero_()


class Status:
    """Device status word {code, detail}."""

    def __init__(self, device: str = "cuda"):
        self.t = torch.zeros(2, dtype=torch.int32, device=device)

    @property
    def ptr(self) -> int:
        return _ptr(self.t)

    def clear(self) -> None:
        self.t.zero_()

    def read(self):
        torch.cuda.synchronize(self.t.device)
        code, detail = (int(v) for v in self.t.cpu().tolist())
        return code, detail

    def check(self, where: str = "device") -> None:
        code, detail = self.read()
        if code:
            raise capi.Csa2Error(code, f"{where} (detail {detail})")


def fp4_compress(x: torch.Tensor, m: int, stream=None):
    """fp32 [groups * m, D] -> FP4 entries of compression rate m (the mean of m rows):
    (codes uint8 [groups, D/2], scales uint8 [groups, D/16])."""
    _need_cuda(x)
    x = x.contiguous()
    D = x.shape[-1]
    groups = x.numel() // D // m
    codes = torch.empty((groups, D // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((groups, D // 16), dtype=torch.uint8, device=x.device)
    check(capi.csa2_fp4_compress(_ptr(x), groups, m, D, _ptr(codes), _ptr(scales), _stream(stream)), "csa2_fp4_compress")
    return codes, scales


def fp4_quantize(x: torch.Tensor, stream=None):
    """fp32 [rows, D] -> (codes uint8 [rows, D/2], scales uint8 [rows, D/16])."""
    _need_cuda(x)
    x = x.contiguous()
    D = x.shape[-1]
    rows = x.numel() // D
    codes = torch.empty(x.shape[:-1] + (D // 2,), dtype=torch.uint8, device=x.device)
    scales = torch.empty(x.shape[:-1] + (D // 16,), dtype=torch.uint8, device=x.device)
    check(capi.csa2_fp4_quantize(_ptr(x), rows, D, _ptr(codes), _ptr(scales), _stream(stream)), "csa2_fp4_quantize")
    return codes, scales


def make_index_args(mode: int, q_pos, qi, w_host: np.ndarray, ki, k: int, P: int = 0, pool_in=None,
                    pool_out=None, topk_out=None, m: int = 0) -> IndexArgs:
    B, Tq, Hi, Di = qi.shape
    a = IndexArgs()
    a.B, a.Tq, a.N, a.Hi, a.Di, a.k, a.P, a.mode = B, Tq, ki.shape[1], Hi, Di, k, P, mode
    a.q_pos, a.qi, a.w, a.ki = _ptr(q_pos), _ptr(qi), w_host.ctypes.data, _ptr(ki)
    a.ki_seq_stride = int(ki.stride(0)) * ki.element_size()
    a.pool_in = _ptr(pool_in)
    a.P_in = 0 if pool_in is None else int(pool_in.shape[-1])
    a.pool_out, a.topk_out = _ptr(pool_out), _ptr(topk_out)
    a.m = m
    return a


def index_topk(mode: str, q_pos, qi, w, ki, k: int, P: int = 0, pool_in=None, ws: Workspace = None,
               status: Status = None, stream=None, m: int = 0):
    """Full or Reindex top-k. Returns (pool or None, topk) as int32 tensors."""
    _need_cuda(q_pos, qi, ki, pool_in)
    mode_id = capi.MODES[mode]
    B, Tq = qi.shape[:2]
    w_host = np.ascontiguousarray(np.asarray(w if not torch.is_tensor(w) else w.cpu().numpy(), dtype=np.int32))
    topk = torch.empty((B, Tq, k), dtype=torch.int32, device=qi.device)
    pool = torch.empty((B, Tq, P), dtype=torch.int32, device=qi.device) if (mode_id == capi.CSA2_FULL and P > 0) else None
    a = make_index_args(mode_id, q_pos, qi, w_host, ki, k, P if mode_id == capi.CSA2_FULL else 0, pool_in, pool,
                        topk, m)
    ws = ws or Workspace(str(qi.device))
    nbytes = capi.csa2_workspace_bytes(0, a)
    buf = ws.get(nbytes)
    st = status.ptr if status is not None else 0
    check(capi.csa2_index_topk(a, _ptr(buf), buf.numel(), st, _stream(stream)), "csa2_index_topk")
    return pool, topk


def make_attn_args(q_pos, q, kv_fp4, kv_scale, topk, kl, vl, local_base, W: int, out, lse, m: int = 0) -> AttnArgs:
    B, Tq, Hq, D = q.shape
    a = AttnArgs()
    a.B, a.Tq, a.N, a.Hq, a.D = B, Tq, kv_fp4.shape[1], Hq, D
    a.k = 0 if topk is None else int(topk.shape[-1])
    a.W = W
    a.Lloc = 0 if kl is None else int(kl.shape[1])
    a.q_pos, a.q, a.kv_fp4, a.kv_scale = _ptr(q_pos), _ptr(q), _ptr(kv_fp4), _ptr(kv_scale)
    a.topk, a.kl, a.vl, a.local_base = _ptr(topk), _ptr(kl), _ptr(vl), _ptr(local_base)
    a.out, a.lse = _ptr(out), _ptr(lse)
    a.m = m
    return a


def sparse_attn(q_pos, q, kv_fp4, kv_scale, topk, kl, vl, local_base, W: int, ws: Workspace = None,
                status: Status = None, stream=None, m: int = 0):
    """Attention over the listed global FP4 rows plus the window. Returns (out bf16, lse fp32)."""
    _need_cuda(q_pos, q, kv_fp4, kv_scale, topk, kl, vl, local_base)
    B, Tq, Hq, D = q.shape
    out = torch.empty((B, Tq, Hq, D), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=q.device)
    a = make_attn_args(q_pos, q, kv_fp4, kv_scale, topk, kl, vl, local_base, W, out, lse, m)
    ws = ws or Workspace(str(q.device))
    buf = ws.get(capi.csa2_workspace_bytes(1, a))
    st = status.ptr if status is not None else 0
    check(capi.csa2_sparse_attn(a, _ptr(buf), buf.numel(), st, _stream(stream)), "csa2_sparse_attn")
    return out, lse


def cache_append(pos, kv_new, kv_fp4, kv_scale, ki_new=None, ki_sets=(), kl_new=None, vl_new=None, kl_layers=(),
                 vl_layers=(), local_base=None, W: int = 0, status: Status = None, stream=None):
    """Append one token per sequence (csa2_cache_append): its global row (fp32 [B, D])
    into the FP4 cache at row pos[b], its index key ([S, B, Di]) into each key set,
    and each layer's local K/V ([L, B, D] bf16) into that layer's buffers
    ([B, Lcap, D]); local_base is updated in place."""
    _need_cuda(pos, kv_new, kv_fp4, kv_scale, ki_new, kl_new, vl_new, local_base, *ki_sets, *kl_layers, *vl_layers)
    a = capi.AppendArgs()
    B, D = kv_new.shape
    a.B, a.N, a.D = B, kv_fp4.shape[1], D
    a.S, a.L, a.W = len(ki_sets), len(kl_layers), W
    a.Di = int(ki_sets[0].shape[-1]) if ki_sets else 0
    a.Lcap = int(kl_layers[0].shape[1]) if kl_layers else 0
    ki_arr = (ctypes.c_void_p * max(1, a.S))(*[_ptr(t) for t in ki_sets])
    kl_arr = (ctypes.c_void_p * max(1, a.L))(*[_ptr(t) for t in kl_layers])
    vl_arr = (ctypes.c_void_p * max(1, a.L))(*[_ptr(t) for t in vl_layers])
    a.pos, a.kv_new, a.kv_fp4, a.kv_scale = _ptr(pos), _ptr(kv_new), _ptr(kv_fp4), _ptr(kv_scale)
    a.ki_new, a.ki = _ptr(ki_new), ctypes.cast(ki_arr, ctypes.c_void_p)
    a.kl_new, a.vl_new = _ptr(kl_new), _ptr(vl_new)
    a.kl, a.vl = ctypes.cast(kl_arr, ctypes.c_void_p), ctypes.cast(vl_arr, ctypes.c_void_p)
    a.local_base = _ptr(local_base)
    st = status.ptr if status is not None else 0
    check(capi.csa2_cache_append(a, st, _stream(stream)), "csa2_cache_append")


def packed_views(specs, device, align: int = 256):
    """One uint8 device buffer holding tensors of the given (shape, dtype) back to
    back, each at an `align`-byte offset, so that a step's inputs or outputs move
    between host and device in one copy. Returns (buffer, views)."""
    sizes, offs, off = [], [], 0
    for shape, dt in specs:
        n = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
        sizes.append(n)
        offs.append(off)
        off = (off + n + align - 1) // align * align
    buf = torch.empty(max(off, align), dtype=torch.uint8, device=device)
    views = [buf[o:o + n].view(dt).view(shape) for (shape, dt), o, n in zip(specs, offs, sizes)]
    return buf, views


class LayerStack:
    """A decoder stack over one shared cache, with its argument structures built once.

    layers: per layer a dict with
      mode 'FULL' | 'REINDEX' | 'REUSE'
      FULL/REINDEX: qi [B,Tq,Hi,Di] int8, w (host ints [Hi]), ki [B,N,Di] int8, k, P (FULL)
      every layer:  q [B,Tq,Hq,D] bf16, kl/vl [B,Lloc,D] bf16, W
    Outputs per layer (allocated here): out, lse; topk for FULL/REINDEX (REUSE layers
    get a copy of their list when keep_reuse_lists=True); pool for FULL with P > 0.
    packed_outputs=True places every out and lse in one device buffer (out_buf).
    """

    def __init__(self, layers: Sequence[Dict], q_pos, kv_fp4, kv_scale, local_base,
                 keep_reuse_lists: bool = False, with_lse: bool = True, packed_outputs: bool = False, m: int = 0):
        dev = q_pos.device
        self.out_buf = None
        packed = None
        if packed_outputs:
            specs = []
            for d in layers:
                B, Tq, Hq, D = d["q"].shape
                specs.append(((B, Tq, Hq, D), torch.bfloat16))
                if with_lse:
                    specs.append(((B, Tq, Hq), torch.float32))
            self.out_buf, packed = packed_views(specs, dev)
            packed = iter(packed)
        self.L = len(layers)
        self.keep = []          # keeps host weight arrays and tensors alive
        self.pools: List[Optional[torch.Tensor]] = []
        self.topks: List[Optional[torch.Tensor]] = []
        self.outs: List[torch.Tensor] = []
        self.lses: List[Optional[torch.Tensor]] = []
        idx_arr = (IndexArgs * self.L)()
        attn_arr = (AttnArgs * self.L)()
        cur_k = 0
        for l, d in enumerate(layers):
            mode = capi.MODES[d["mode"]]
            q = d["q"]
            B, Tq, Hq, D = q.shape
            pool = topk = None
            if mode in (capi.CSA2_FULL, capi.CSA2_REINDEX):
                w_host = np.ascontiguousarray(np.asarray(d["w"], dtype=np.int32))
                self.keep.append(w_host)
                P = int(d.get("P", 0)) if mode == capi.CSA2_FULL else 0
                cur_k = int(d["k"])
                topk = torch.empty((B, Tq, cur_k), dtype=torch.int32, device=dev)
                if P > 0:
                    pool = torch.empty((B, Tq, P), dtype=torch.int32, device=dev)
                idx_arr[l] = make_index_args(mode, q_pos, d["qi"], w_host, d["ki"], cur_k, P, None, pool, topk, m)
            else:
                if keep_reuse_lists:
                    topk = torch.empty((B, Tq, cur_k), dtype=torch.int32, device=dev)
                a = IndexArgs()
                a.mode = mode
                a.topk_out = _ptr(topk)
                idx_arr[l] = a
            if packed is not None:
                out = next(packed)
                lse = next(packed) if with_lse else None
            else:
                out = torch.empty((B, Tq, Hq, D), dtype=torch.bfloat16, device=dev)
                lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=dev) if with_lse else None
            kl, vl = d.get("kl"), d.get("vl")
            attn_arr[l] = make_attn_args(q_pos, q, kv_fp4, kv_scale, None, kl, vl, local_base, int(d["W"]), out, lse,
                                         m)
            self.keep.extend([d.get("qi"), d.get("ki"), q, kl, vl])
            self.pools.append(pool)
            self.topks.append(topk)
            self.outs.append(out)
            self.lses.append(lse)
        self.keep.extend([q_pos, kv_fp4, kv_scale, local_base])
        self.idx_arr, self.attn_arr = idx_arr, attn_arr
        self.args = StackArgs(self.L, idx_arr, attn_arr)
        self.ws_bytes = capi.csa2_workspace_bytes(2, self.args)
        if self.ws_bytes == 0:
            raise ValueError("invalid layer stack arguments")

    def run(self, ws: Workspace, status: Status = None, stream=None) -> None:
        buf = ws.get(self.ws_bytes)
        st = status.ptr if status is not None else 0
        check(capi.csa2_layer_stack(self.args, _ptr(buf), buf.numel(), st, _stream(stream)), "csa2_layer_stack")

    def run_raw(self, ws_ptr: int, ws_bytes: int, status_ptr: int, stream_ptr: int) -> int:
        """The bare C call, for tight timing loops (returns the status code)."""
        return capi.lib().csa2_layer_stack(self.args, ws_ptr, ws_bytes, status_ptr, stream_ptr)
