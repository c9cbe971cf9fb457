"""Helpers shared by the GPU tests: move a synthetic workload to the device and
compare the CUDA path with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import csa2_oracle as O
from sparse_attention_shared_b200 import ops

OUT_TOL = 3e-3      # max |out_gpu(bf16) - out_oracle(fp64)|
LSE_TOL = 1e-3


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return dev(bits.view(np.int16), torch.bfloat16)


class DeviceWorkload:
    """A synth workload's tensors on the GPU, with the cache quantised by the CUDA path."""

    def __init__(self, wl, status=None):
        self.wl = wl
        s = wl.spec
        self.q_pos = dev(wl.q_pos())
        self.local_base = dev(wl.local_base_arr())
        kv = dev(wl.kv_f32())
        if s.m > 1:
            self.kv_fp4, self.kv_scale = ops.fp4_compress(kv.view(-1, s.D), s.m)
        else:
            self.kv_fp4, self.kv_scale = ops.fp4_quantize(kv.view(-1, s.D))
        self.kv_fp4 = self.kv_fp4.view(s.B, s.N, s.D // 2)
        self.kv_scale = self.kv_scale.view(s.B, s.N, s.D // 16)
        del kv
        self.ki = {}
        for l in s.layers:
            if l.key_set >= 0 and l.key_set not in self.ki:
                self.ki[l.key_set] = dev(wl.ki(l.key_set))

    def layer_dicts(self):
        s, wl = self.wl.spec, self.wl
        out = []
        for li, L in enumerate(s.layers):
            d = {"mode": L.mode, "q": bf16_dev(wl.q(li)), "kl": bf16_dev(wl.kl(li)), "vl": bf16_dev(wl.vl(li)),
                 "W": s.W}
            if L.mode in ("FULL", "REINDEX"):
                d.update(qi=dev(wl.qi(li)), w=wl.w(li), ki=self.ki[L.key_set], k=L.k, P=L.P)
            out.append(d)
        return out


def assert_list_invariants(lists: np.ndarray, q_pos: np.ndarray, what: str):
    """Every list [..., len] of a query at position t holds distinct positions in
    [0, t], ascending, with -1 only as padding at the tail ([CED] Fig. 2: causal
    access; the lists' order and padding are this library's layout)."""
    g = np.asarray(lists)
    t = np.asarray(q_pos).reshape(g.shape[:-1] + (1,))
    valid = g >= 0
    assert np.all(valid[..., 1:] <= valid[..., :-1]), f"{what}: -1 before a valid entry"
    assert np.all(g[valid] <= np.broadcast_to(t, g.shape)[valid]), f"{what}: an entry past the query position"
    inc = (g[..., 1:] > g[..., :-1]) | ~valid[..., 1:]
    assert np.all(inc), f"{what}: entries not strictly ascending"


def assert_lists_equal(gpu: torch.Tensor, ref: np.ndarray, what: str):
    g = gpu.cpu().numpy()
    if not np.array_equal(g, ref):
        bad = np.argwhere(g != ref)
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {bad[:5].tolist()}: "
                             f"gpu {g[tuple(bad[0])]} oracle {ref[tuple(bad[0])]}")


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |x|: the largest error of rounding x to bf16."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.ldexp(1.0, (e - 8).astype(np.int64)), 0.0)


def assert_attn_close(out: torch.Tensor, lse, ref_out: np.ndarray, ref_lse: np.ndarray, what: str,
                      output_rounding: bool = False):
    """max |out - ref| <= 3e-3 (the bar for the five workloads). With output_rounding,
    the bar applies to the error beyond the bf16 output's own rounding (half a bf16 ulp
    of the reference): an output of magnitude >= 1 cannot be within 3e-3 of its fp64
    value once stored as bf16 (half an ulp there is 3.9e-3)."""
    o = out.float().cpu().numpy().astype(np.float64)
    diff = np.abs(o - ref_out)
    if output_rounding:
        diff = np.maximum(diff - bf16_half_ulp(ref_out), 0.0)
    err = diff.max()
    assert err <= OUT_TOL, f"{what}: max |out diff| {err:.3e} > {OUT_TOL}"
    if lse is not None:
        l = lse.cpu().numpy().astype(np.float64)
        e2 = np.abs(l - ref_lse).max()
        assert e2 <= LSE_TOL, f"{what}: max |lse diff| {e2:.3e} > {LSE_TOL}"
    return err
