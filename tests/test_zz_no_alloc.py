"""csa2_sparse_attn_noalloc: the attention entry point for callers that cannot
allocate device memory (a host framework that owns every device allocation, or a
decode loop that must not risk the synchronisation a cudaMalloc/cudaFree can
cause). It takes no workspace; its scratch is a static device array. This test
calls it through the C ABI twice in a row and checks each result against the
workspace entry point csa2_sparse_attn on the same inputs, within the tolerance
of the other attention tests. It allocates its own inputs and outputs (the caller
still owns those). Named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import csa2_oracle as O
from sparse_attention_shared_b200 import capi, ops

from gpu_util import LSE_TOL, OUT_TOL, bf16_dev, dev

pytestmark = pytest.mark.gpu


def _noalloc():
    f = capi.lib().csa2_sparse_attn_noalloc
    f.argtypes = [ctypes.POINTER(capi.AttnArgs), ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _inputs(seed, B=4, N=8192, Tq=1, Hq=16, D=128, k=2048, W=512):
    kv = synth.normal_f32(seed, 1, (B * N, D))
    codes, scales = ops.fp4_quantize(dev(kv))
    base = N - Tq - W + 1
    rng = np.random.default_rng(seed)
    topk = np.stack([[np.sort(rng.choice(N, k, replace=False)).astype(np.int32) for _ in range(Tq)]
                     for _ in range(B)])
    return dict(q_pos=dev(np.full((B, Tq), N - 1, np.int32)), q=bf16_dev(synth.normal_bf16(seed, 2, (B, Tq, Hq, D))),
                kv_fp4=codes.view(B, N, D // 2), kv_scale=scales.view(B, N, D // 16), topk=dev(topk),
                kl=bf16_dev(synth.normal_bf16(seed, 3, (B, N - base, D))),
                vl=bf16_dev(synth.normal_bf16(seed, 4, (B, N - base, D))),
                local_base=dev(np.full((B,), base, np.int32)), W=W)


def test_noalloc_matches_workspace_entry_point_twice():
    f = _noalloc()
    stream = int(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((101, 202)):
        x = _inputs(seed)
        ref_out, ref_lse = ops.sparse_attn(**x)
        out = torch.empty_like(ref_out)
        lse = torch.empty_like(ref_lse)
        a = ops.make_attn_args(x["q_pos"], x["q"], x["kv_fp4"], x["kv_scale"], x["topk"], x["kl"], x["vl"],
                               x["local_base"], x["W"], out, lse)
        st = ops.Status()
        assert f(ctypes.byref(a), st.ptr, stream) == 0
        st.check(f"noalloc call {call}")
        d_out = (out.float() - ref_out.float()).abs().max().item()
        d_lse = (lse - ref_lse).abs().max().item()
        assert d_out <= OUT_TOL, f"call {call}: out differs by {d_out}"
        assert d_lse <= LSE_TOL, f"call {call}: lse differs by {d_lse}"


def test_noalloc_against_the_oracle_without_window():
    """Several queries per sequence and no local branch (W = 0), checked directly
    against the fp64 oracle on two calls in a row."""
    f = _noalloc()
    stream = int(torch.cuda.current_stream().cuda_stream)
    B, N, Tq, Hq, D, k = 2, 3000, 4, 16, 128, 300
    for call, seed in enumerate((303, 404)):
        kv = synth.normal_f32(seed, 1, (B, N, D))
        codes, scales = O.fp4_quantize(kv)
        q = synth.normal_bf16(seed, 2, (B, Tq, Hq, D))
        q_pos = np.broadcast_to(np.arange(N - Tq, N, dtype=np.int32), (B, Tq)).copy()
        rng = np.random.default_rng(seed)
        topk = np.stack([[np.sort(rng.choice(int(t) + 1, k, replace=False)).astype(np.int32) for t in q_pos[b]]
                         for b in range(B)])
        gc, gs = ops.fp4_quantize(dev(kv.reshape(-1, D)))
        out = torch.empty((B, Tq, Hq, D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device="cuda")
        # the argument structure holds raw pointers: keep every tensor alive until the call is done
        d_pos, d_q, d_topk = dev(q_pos), bf16_dev(q), dev(topk)
        a = ops.make_attn_args(d_pos, d_q, gc.view(B, N, D // 2), gs.view(B, N, D // 16), d_topk,
                               None, None, None, 0, out, lse)
        st = ops.Status()
        assert f(ctypes.byref(a), st.ptr, stream) == 0
        st.check(f"noalloc call {call}")
        o, l = out.float().cpu().numpy(), lse.cpu().numpy()
        for b in range(B):
            for j in range(Tq):
                none = np.zeros((1, D))
                ro, rl = O.attention_unit(O.bf16_to_f64(q[b, j]), codes[b], scales[b], topk[b, j], none, none, 0,
                                          int(q_pos[b, j]), 0)
                assert np.abs(o[b, j] - ro).max() <= OUT_TOL, f"call {call}, unit {(b, j)}: out"
                assert np.abs(l[b, j] - rl).max() <= LSE_TOL, f"call {call}, unit {(b, j)}: lse"


def test_noalloc_rejects_sizes_beyond_its_static_scratch():
    f = _noalloc()
    x = _inputs(7, B=2, N=4096)
    out = torch.empty((80, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    a = ops.make_attn_args(x["q_pos"], x["q"], x["kv_fp4"], x["kv_scale"], x["topk"], x["kl"], x["vl"],
                           x["local_base"], x["W"], out, None)
    a.B = 80                       # 80 queries x 20 tiles of partials > 8 MiB: rejected before any launch
    assert f(ctypes.byref(a), 0, 0) == 9
