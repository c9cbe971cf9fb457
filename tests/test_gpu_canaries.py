"""Guard bands around every output of a layer stack.

Each output buffer (pool, top-k list, bf16 out, fp32 lse of every layer) is carved
from a larger allocation whose bytes before and after it hold a known pattern.
After the call the patterns must be intact: no kernel writes outside the buffers
the caller passed. The workloads are small enough to run in seconds but cover the
Full and Reindex kernels (scores in shared memory and spilled), the multi-query
scoring kernel, the cluster attention and the ticket merge."""
import numpy as np
import pytest
import torch

import synth
from sparse_attention_shared_b200 import ops

from gpu_util import DeviceWorkload

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side
PATTERN = 0xA5


class Guarded:
    """Tensors carved out of byte buffers with guard bands on both sides."""

    def __init__(self):
        self.bufs = []

    def empty(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.bufs.append((raw, n))
        return raw[GUARD:GUARD + n].view(dtype).view(shape)

    def check(self):
        torch.cuda.synchronize()
        for raw, n in self.bufs:
            head = raw[:GUARD].cpu().numpy()
            tail = raw[GUARD + n:].cpu().numpy()
            assert (head == PATTERN).all() and (tail == PATTERN).all(), "a guard band was overwritten"


def _guarded_stack(wl):
    s = wl.spec
    dw = DeviceWorkload(wl)
    st = ops.LayerStack(dw.layer_dicts(), dw.q_pos, dw.kv_fp4, dw.kv_scale, dw.local_base, keep_reuse_lists=True,
                        m=s.m)
    g = Guarded()
    # re-point every output of the argument structures at guarded buffers
    for l in range(st.L):
        ia, aa = st.idx_arr[l], st.attn_arr[l]
        if st.topks[l] is not None:
            st.topks[l] = g.empty(tuple(st.topks[l].shape), torch.int32)
            ia.topk_out = st.topks[l].data_ptr()
        if st.pools[l] is not None:
            st.pools[l] = g.empty(tuple(st.pools[l].shape), torch.int32)
            ia.pool_out = st.pools[l].data_ptr()
        st.outs[l] = g.empty(tuple(st.outs[l].shape), torch.bfloat16)
        aa.out = st.outs[l].data_ptr()
        st.lses[l] = g.empty(tuple(st.lses[l].shape), torch.float32)
        aa.lse = st.lses[l].data_ptr()
    return st, g


@pytest.mark.parametrize("name,kw", [
    ("stack20_128k", dict(B=3, N=20000)),                    # Full, Reindex, cluster attention
    ("paper_schedule", dict(B=2, N=9000)),
    ("long_1m", dict(N=40000, Tq=6)),                        # shared-key sample, estimate, mark and cut
    ("decode_full", dict(B=150, N=20000)),                   # more units than SMs: one CTA per unit, spilled scores
    ("replay_prefill", dict(B=1, N=9000, Tq=160, W=128)),    # shared-key cut and Reindex cut, one CTA per query
])
def test_outputs_stay_inside_their_buffers(name, kw):
    wl = synth.make_workload(name, **kw)
    st, g = _guarded_stack(wl)
    ws, status = ops.Workspace(), ops.Status()
    st.run(ws, status)
    status.check(name)
    g.check()


def test_ticket_attention_stays_inside_its_buffers():
    B, N, D, Hq, k, W = 2, 8192, 128, 16, 4096, 2048           # 16 window tiles: more than one cluster holds
    kv = synth.normal_f32(3, 1, (B * N, D))
    codes, scales = ops.fp4_quantize(torch.from_numpy(kv).cuda())
    rng = np.random.default_rng(3)
    topk = np.stack([[np.sort(rng.choice(N, k, replace=False)).astype(np.int32)] for _ in range(B)])
    base = N - W
    g = Guarded()
    out = g.empty((B, 1, Hq, D), torch.bfloat16)
    lse = g.empty((B, 1, Hq), torch.float32)
    q = torch.from_numpy(synth.normal_bf16(3, 2, (B, 1, Hq, D)).view(np.int16)).cuda().view(torch.bfloat16)
    kl = torch.from_numpy(synth.normal_bf16(3, 3, (B, W, D)).view(np.int16)).cuda().view(torch.bfloat16)
    vl = torch.from_numpy(synth.normal_bf16(3, 4, (B, W, D)).view(np.int16)).cuda().view(torch.bfloat16)
    # the argument structure holds raw pointers: keep every tensor alive until the call is done
    d_pos = torch.full((B, 1), N - 1, dtype=torch.int32, device="cuda")
    d_topk = torch.from_numpy(topk).cuda()
    d_base = torch.full((B,), base, dtype=torch.int32, device="cuda")
    a = ops.make_attn_args(d_pos, q, codes.view(B, N, D // 2), scales.view(B, N, D // 16), d_topk, kl, vl, d_base, W,
                           out, lse)
    from sparse_attention_shared_b200 import capi
    ws, status = ops.Workspace(), ops.Status()
    buf = ws.get(capi.csa2_workspace_bytes(1, a))
    capi.check(capi.csa2_sparse_attn(a, buf.data_ptr(), buf.numel(), status.ptr,
                                     int(torch.cuda.current_stream().cuda_stream)), "attention")
    status.check("ticket attention")
    g.check()
