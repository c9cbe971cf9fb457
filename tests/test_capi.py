"""The C-ABI library without a GPU: it builds for sm_100a, loads, exports every
entry point that include/csa2.h declares, and rejects bad arguments on the host
before launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest

from sparse_attention_shared_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(csa2_\w+)\s*\(", txt))
    return names


def test_library_exports_every_declared_symbol():
    L = capi.lib()
    declared = _declared()
    assert {"csa2_index_topk", "csa2_sparse_attn", "csa2_layer_stack", "csa2_fp4_quantize",
            "csa2_workspace_bytes", "csa2_status_string"} <= declared
    for name in declared:
        assert hasattr(L, name), name


def test_phase_trace_build_exports_its_buffers_entry_points():
    """The phase-trace variant (-DCSA2_PHASE_TRACE) has every declared entry point plus
    the two trace-buffer setters; the normal library has no trace code."""
    import ctypes
    from sparse_attention_shared_b200 import build
    T = ctypes.CDLL(build.build(trace=True))
    for name in _declared() | {"csa2_trace_set_idx", "csa2_trace_set_attn"}:
        assert hasattr(T, name), name
    L = capi.lib()
    assert not hasattr(L, "csa2_trace_set_idx") and not hasattr(L, "csa2_trace_set_attn")


def test_wait_controls_validation():
    assert capi.csa2_set_wait_controls(-1, 0) == 2      # CSA2_ERR_SHAPE
    assert capi.csa2_set_wait_controls(0, 0) == 0       # the default budget, no injection


def test_status_strings():
    for code in range(10):
        assert capi.csa2_status_string(code)


def _index_args(**kw):
    a = capi.IndexArgs()
    a.B, a.Tq, a.N, a.Hi, a.Di, a.k, a.P, a.mode = 1, 1, 1024, 8, 64, 16, 64, capi.CSA2_FULL
    fake = 1 << 20       # aligned, never dereferenced: validation fails or no workspace is given
    w = np.ones(8, np.int32)
    a.q_pos = a.qi = a.ki = a.topk_out = a.pool_out = fake
    a.w = w.ctypes.data
    a.ki_seq_stride = 1024 * 64
    for k, v in kw.items():
        setattr(a, k, v)
    return a, w


@pytest.mark.parametrize("field,value,code", [
    ("q_pos", 0, 1), ("Hi", 17, 2), ("Di", 24, 2), ("k", 0, 2), ("k", 65, 2), ("N", 1 << 27, 2),
    ("ki_seq_stride", 1000, 3), ("qi", (1 << 20) + 4, 3), ("mode", 2, 4), ("pool_out", 0, 1),
])
def test_index_validation(field, value, code):
    a, _w = _index_args(**{field: value})
    assert capi.csa2_index_topk(a, 0, 0, 0, 0) == code


def test_index_weight_bound_and_workspace():
    a, w = _index_args()
    w[:] = 300                                   # 8 * 300 * 64 * 16384 >= 2^31
    assert capi.csa2_index_topk(a, 0, 0, 0, 0) == 5
    a, w = _index_args()
    assert capi.csa2_workspace_bytes(0, a) > 0
    assert capi.csa2_index_topk(a, 0, 0, 0, 0) == 9          # no workspace


def test_attn_validation():
    a = capi.AttnArgs()
    a.B, a.Tq, a.N, a.Hq, a.D, a.k, a.W, a.Lloc = 1, 1, 1024, 16, 128, 64, 128, 128
    fake = 1 << 20
    a.q_pos = a.q = a.kv_fp4 = a.kv_scale = a.topk = a.kl = a.vl = a.local_base = a.out = fake
    assert capi.csa2_workspace_bytes(1, a) > 0
    assert capi.csa2_sparse_attn(a, 0, 0, 0, 0) == 9
    a.D = 96
    assert capi.csa2_sparse_attn(a, 0, 0, 0, 0) == 6
    a.D, a.Hq = 128, 33
    assert capi.csa2_sparse_attn(a, 0, 0, 0, 0) == 6
    a.Hq, a.kl = 16, 0
    assert capi.csa2_sparse_attn(a, 0, 0, 0, 0) == 1


def test_stack_mode_order():
    ia, _w = _index_args()
    aa = capi.AttnArgs()
    aa.B, aa.Tq, aa.N, aa.Hq, aa.D, aa.W = 1, 1, 1024, 16, 128, 0
    aa.q_pos = aa.q = aa.kv_fp4 = aa.kv_scale = aa.out = 1 << 20
    reuse = capi.IndexArgs()
    reuse.mode = capi.CSA2_REUSE
    idx = (capi.IndexArgs * 2)(reuse, ia)
    att = (capi.AttnArgs * 2)(aa, aa)
    assert capi.csa2_layer_stack(capi.StackArgs(2, idx, att), 0, 0, 0, 0) == 4
    idx = (capi.IndexArgs * 2)(ia, reuse)
    s = capi.StackArgs(2, idx, att)
    assert capi.csa2_workspace_bytes(2, s) > 0
    assert capi.csa2_layer_stack(s, 0, 0, 0, 0) == 9
    ri = capi.IndexArgs.from_buffer_copy(ia)
    ri.mode = capi.CSA2_REINDEX
    ia0 = capi.IndexArgs.from_buffer_copy(ia)
    ia0.P = 0
    idx = (capi.IndexArgs * 2)(ia0, ri)          # REINDEX without a pool
    assert capi.csa2_layer_stack(capi.StackArgs(2, idx, att), 0, 0, 0, 0) == 4


def _shared_key_scratch(units, N, sms=148):
    """The shared-key path's scratch, restated: the fallback's spill (up to 16 queries at a
    time, groups of G CTAs each over the SMs, at most 64 MB), the sampled tiles' scores (32 to 128 tiles of 128
    positions a query, at least one tile in 64), one candidate word per 32 positions a
    query, the estimates and the fallback list; each part rounded up to 256 bytes."""
    a256 = lambda x: (x + 255) // 256 * 256
    ntile = -(-N // 128)
    want = min(128, max(32, -(-ntile // 64)))
    tstep = max(1, -(-ntile // want))
    sstride = -(-ntile // tstep) * 128
    groups = max(1, min(16, units, (64 << 20) // (a256(N) * 4)))
    G = max(1, min(64, sms // groups, (N + 1023) // 1024))
    chunk = a256(-(-N // G))
    spill = a256(groups * G * chunk * 4 + 512) if chunk > 16384 else 0
    return spill + a256(units * sstride * 4) + a256(units * ntile * 4 * 4) + a256(units * 16) + a256((units + 1) * 4)


def test_index_workspace_of_the_shared_key_path():
    """A Full call with at least 4 queries per sequence on a key set of at least 8192
    positions scores its queries in blocks and keeps no query's scores in full: its
    workspace holds a sample, candidate words, estimates and the fallback's spill, well
    below B*Tq*N int32 scores; smaller calls score one query per unit and need none."""
    def ws(Tq, N):
        a, _w = _index_args(Tq=Tq, N=N, ki_seq_stride=N * 64)
        return capi.csa2_workspace_bytes(0, a)
    base = ws(1, 8192)
    for Tq, N in [(64, 1 << 20), (64, 8192), (4, 8192), (4096, 69632)]:
        extra = ws(Tq, N) - base
        assert extra == _shared_key_scratch(Tq, N), (Tq, N)
        if N >= 69632:
            assert extra < Tq * N * 4 // 2, (Tq, N)
    assert ws(64, 4096) == base      # below 8192 keys
    assert ws(3, 8192) == base       # fewer than 4 queries


def test_compress_validation():
    fake = 1 << 20
    assert capi.csa2_fp4_compress(fake, 4, 3, 128, fake, fake, 0) == 2     # m must be 1, 2, 4 or 8
    assert capi.csa2_fp4_compress(fake, 4, 2, 24, fake, fake, 0) == 2      # D % 16
    assert capi.csa2_fp4_compress(0, 4, 2, 128, fake, fake, 0) == 1
    assert capi.csa2_fp4_compress(fake + 4, 4, 2, 128, fake, fake, 0) == 3


def test_compression_rate_field_is_validated():
    a, _w = _index_args(m=9)
    assert capi.csa2_index_topk(a, 0, 0, 0, 0) == 2
    a, _w = _index_args(m=2)
    assert capi.csa2_workspace_bytes(0, a) > 0


def test_append_validation():
    fake = 1 << 20
    arr = (ctypes.c_void_p * 2)(fake, fake)

    def args(**kw):
        a = capi.AppendArgs()
        a.B, a.N, a.D, a.Di, a.S, a.L, a.W, a.Lcap = 2, 1024, 128, 64, 1, 2, 64, 127
        a.pos = a.kv_new = a.kv_fp4 = a.kv_scale = a.ki_new = a.kl_new = a.vl_new = a.local_base = fake
        a.ki = a.kl = a.vl = ctypes.cast(arr, ctypes.c_void_p).value
        for k, v in kw.items():
            setattr(a, k, v)
        return a
    assert capi.csa2_cache_append(args(Lcap=126), 0, 0) == 2      # Lcap < 2W - 1
    assert capi.csa2_cache_append(args(S=33), 0, 0) == 2
    assert capi.csa2_cache_append(args(D=120), 0, 0) == 2
    assert capi.csa2_cache_append(args(pos=0), 0, 0) == 1
    assert capi.csa2_cache_append(args(kv_new=fake + 8), 0, 0) == 3
    assert capi.csa2_cache_append(args(L=1, W=0), 0, 0) == 2
