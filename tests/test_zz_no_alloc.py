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


def test_noalloc_rejects_sizes_beyond_its_static_scratch():
    f = _noalloc()
    x = _inputs(7, B=2, N=4096)
    out = torch.empty((80, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    a = ops.make_attn_args(x["q_pos"], x["q"], x["kv_fp4"], x["kv_scale"], x["topk"], x["kl"], x["vl"],
                           x["local_base"], x["W"], out, None)
    a.B = 80                       # 80 queries x 20 tiles of partials > 8 MiB: rejected before any launch
    assert f(ctypes.byref(a), 0, 0) == 9
