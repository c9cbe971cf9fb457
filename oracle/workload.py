"""Run the oracle on a synthetic workload, one (sequence, query) unit at a time.

TEST INFRASTRUCTURE (see csa2_oracle.py): used only by the tests, smoke() and
the CPU baseline leg of the benchmark.
"""
from __future__ import annotations

from typing import Dict, Iterable, List, Tuple

import numpy as np

from . import csa2_oracle as O


class OracleCache:
    """Per-sequence FP4 quantisation of a workload's global KV, done by the oracle."""

    def __init__(self, wl):
        self.wl = wl
        self._seq: Dict[int, Tuple[np.ndarray, np.ndarray]] = {}

    def seq(self, b: int):
        if b not in self._seq:
            m = self.wl.spec.m
            x = self.wl.kv_f32()[b]
            self._seq[b] = O.fp4_quantize(O.compress_entries(x, m) if m > 1 else x)
        return self._seq[b]


def layer_inputs(wl, b: int, j: int, with_attention: bool = True) -> List[dict]:
    """The oracle's per-layer argument dicts for query j of sequence b."""
    s = wl.spec
    out = []
    for li, L in enumerate(s.layers):
        d = {"mode": L.mode}
        if L.mode in (O.FULL, O.REINDEX):
            d.update(qi=wl.qi(li)[b, j], w=wl.w(li), keys=wl.ki(L.key_set)[b], k=L.k, P=L.P)
        if with_attention:
            d.update(q=O.bf16_to_f64(wl.q(li)[b, j]), kl=O.bf16_to_f64(wl.kl(li)[b]),
                     vl=O.bf16_to_f64(wl.vl(li)[b]), W=s.W)
        out.append(d)
    return out


def run_units(wl, units: Iterable[Tuple[int, int]], cache: OracleCache = None,
              with_attention: bool = True) -> Dict[Tuple[int, int], List[dict]]:
    """Oracle results for the given (b, j) units: per layer {mode, pool, topk, out, lse}."""
    cache = cache or OracleCache(wl)
    res = {}
    for b, j in units:
        t = int(wl.q_pos()[b, j])
        codes, scales = cache.seq(b) if with_attention else (None, None)
        res[(b, j)] = O.layer_stack_unit(layer_inputs(wl, b, j, with_attention), t, codes, scales,
                                         int(wl.local_base_arr()[b]), with_attention, wl.spec.m)
    return res
