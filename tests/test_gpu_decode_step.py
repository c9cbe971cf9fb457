"""Decode steps end to end: csa2_cache_append, then the layer stack, token after token.

"CED: Continuing Context with a Causal Encoder and Decoder", "Why Prefill
Recomputes a Recent Segment" (closing paragraph): after each output the new
token's global KV is appended to the shared cache and each layer updates its
local state; the next token's layers then read the grown cache. Here six tokens
are appended one at a time to three sequences whose local buffers refill at
different steps. After every append the device cache, keys and local buffers are
checked against the histories they came from (the global rows bit for bit against
the oracle's quantiser), and the stack's lists and outputs for the new token
against the oracle run directly on the full histories: keys and cache rows
0..p, and the window [p - W + 1, p] of each layer's local history."""
import numpy as np
import pytest
import torch

import synth
from oracle import cpp as C
from oracle import csa2_oracle as O
from sparse_attention_shared_b200 import ops

from gpu_util import assert_attn_close, assert_lists_equal, bf16_dev, dev

pytestmark = pytest.mark.gpu

B, NCAP, N0, D, Di, Hq, Hi, W = 3, 6000, 5000, 128, 64, 16, 8, 64
LCAP = 2 * W - 1
STEPS = 6
LAYERS = [dict(mode="FULL", k=256, P=1024, key_set=0), dict(mode="REUSE"), dict(mode="REINDEX", k=256, key_set=1),
          dict(mode="REUSE")]


def _bits_to_dev(bits):
    return bf16_dev(np.ascontiguousarray(bits))


def test_append_then_stack_six_tokens():
    seed = 41
    kv_hist = synth.normal_f32(seed, 1, (B, NCAP, D))
    keys_hist = [synth.randint_i8(seed, 2 + s, (B, NCAP, Di)) for s in range(2)]
    kl_hist = [synth.normal_bf16(seed, 10 + l, (B, NCAP, D)) for l in range(len(LAYERS))]
    vl_hist = [synth.normal_bf16(seed, 30 + l, (B, NCAP, D)) for l in range(len(LAYERS))]
    base0 = np.array([N0 - 124 + b for b in range(B)], np.int32)      # sequence b refills one step earlier

    # initial device state: positions [0, N0) in the cache and keys, [base0, N0) in the local buffers
    ws, st = ops.Workspace(), ops.Status()
    codes = torch.zeros((B, NCAP, D // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((B, NCAP, D // 16), dtype=torch.uint8, device="cuda")
    c0, s0 = ops.fp4_quantize(dev(np.ascontiguousarray(kv_hist[:, :N0]).reshape(-1, D)))
    codes[:, :N0] = c0.view(B, N0, D // 2)
    scales[:, :N0] = s0.view(B, N0, D // 16)
    keys = [torch.zeros((B, NCAP, Di), dtype=torch.int8, device="cuda") for _ in range(2)]
    for s in range(2):
        keys[s][:, :N0] = dev(np.ascontiguousarray(keys_hist[s][:, :N0]))
    kl = [torch.zeros((B, LCAP, D), dtype=torch.bfloat16, device="cuda") for _ in LAYERS]
    vl = [torch.zeros((B, LCAP, D), dtype=torch.bfloat16, device="cuda") for _ in LAYERS]
    for l in range(len(LAYERS)):
        for b in range(B):
            n = N0 - int(base0[b])
            kl[l][b, :n] = _bits_to_dev(kl_hist[l][b, base0[b]:N0])
            vl[l][b, :n] = _bits_to_dev(vl_hist[l][b, base0[b]:N0])
    base = dev(base0)
    w = [synth.randint_i32(seed, 50 + l, (Hi,), 1, 8) for l in range(len(LAYERS))]

    for i in range(STEPS):
        p = N0 + i
        pos = dev(np.full((B,), p, np.int32))
        ops.cache_append(pos, dev(np.ascontiguousarray(kv_hist[:, p])), codes, scales,
                         ki_new=dev(np.stack([keys_hist[s][:, p] for s in range(2)])), ki_sets=keys,
                         kl_new=_bits_to_dev(np.stack([kl_hist[l][:, p] for l in range(len(LAYERS))])),
                         vl_new=_bits_to_dev(np.stack([vl_hist[l][:, p] for l in range(len(LAYERS))])),
                         kl_layers=kl, vl_layers=vl, local_base=base, W=W, status=st)
        st.check(f"append {i}")
        # the state after the append
        rc, rs = C.fp4_quantize(np.ascontiguousarray(kv_hist[:, : p + 1]))
        assert_lists_equal(codes[:, : p + 1], rc, f"step {i}: FP4 codes")
        assert_lists_equal(scales[:, : p + 1], rs, f"step {i}: E4M3 scales")
        for s in range(2):
            assert_lists_equal(keys[s][:, : p + 1], keys_hist[s][:, : p + 1], f"step {i}: key set {s}")
        bh = base.cpu().numpy()
        for b in range(B):
            assert p - bh[b] < LCAP and bh[b] <= p - W + 1
            lo = p - W + 1
            for l in range(len(LAYERS)):
                got_k = kl[l][b, lo - bh[b]: p - bh[b] + 1].view(torch.int16).cpu().numpy().view(np.uint16)
                got_v = vl[l][b, lo - bh[b]: p - bh[b] + 1].view(torch.int16).cpu().numpy().view(np.uint16)
                assert np.array_equal(got_k, kl_hist[l][b, lo: p + 1]), f"step {i} layer {l} seq {b}: local K"
                assert np.array_equal(got_v, vl_hist[l][b, lo: p + 1]), f"step {i} layer {l} seq {b}: local V"

        # the new token through the stack, against the oracle on the full histories
        q = [synth.normal_bf16(seed + i, 60 + l, (B, 1, Hq, D)) for l in range(len(LAYERS))]
        qi = [synth.randint_i8(seed + i, 80 + l, (B, 1, Hi, Di)) for l in range(len(LAYERS))]
        layers = []
        for l, L in enumerate(LAYERS):
            d = {"mode": L["mode"], "q": _bits_to_dev(q[l]), "kl": kl[l], "vl": vl[l], "W": W}
            if L["mode"] != "REUSE":
                d.update(qi=dev(qi[l]), w=w[l], ki=keys[L["key_set"]], k=L["k"], P=L.get("P", 0))
            layers.append(d)
        stack = ops.LayerStack(layers, dev(np.full((B, 1), p, np.int32)), codes, scales, base, keep_reuse_lists=True)
        stack.run(ws, st)
        torch.cuda.synchronize()
        st.check(f"stack {i}")
        for b in range(B):
            cur = pool = None
            for l, L in enumerate(LAYERS):
                if L["mode"] == "FULL":
                    pool, cur = C.index_full(qi[l][b, 0], w[l], keys_hist[L["key_set"]][b, : p + 1], p, L["k"], L["P"])
                    assert_lists_equal(stack.pools[l][b, 0], pool, f"step {i} layer {l} seq {b}: pool")
                elif L["mode"] == "REINDEX":
                    cur = C.index_reindex(qi[l][b, 0], w[l], keys_hist[L["key_set"]][b, : p + 1], pool, L["k"])
                assert_lists_equal(stack.topks[l][b, 0], cur, f"step {i} layer {l} seq {b}: list")
                ro, rl = C.attention_unit(q[l][b, 0], rc[b], rs[b], cur, kl_hist[l][b], vl_hist[l][b], 0, p, W)
                # window 64 and top-256 give outputs up to about 1.5 here: the bar applies beyond
                # the bf16 output's own rounding
                assert_attn_close(stack.outs[l][b, 0], stack.lses[l][b, 0], ro, rl, f"step {i} layer {l} seq {b}",
                                  output_rounding=True)


def test_append_rejects_bad_sizes():
    from sparse_attention_shared_b200 import capi
    pos = dev(np.zeros((1,), np.int32))
    kv = torch.zeros((1, D), dtype=torch.float32, device="cuda")
    codes = torch.zeros((1, 8, D // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((1, 8, D // 16), dtype=torch.uint8, device="cuda")
    kl = [torch.zeros((1, 2 * W - 2, D), dtype=torch.bfloat16, device="cuda")]    # one row short of 2W - 1
    with pytest.raises(capi.Csa2Error) as e:
        ops.cache_append(pos, kv, codes, scales, kl_new=torch.zeros((1, 1, D), dtype=torch.bfloat16, device="cuda"),
                         vl_new=torch.zeros((1, 1, D), dtype=torch.bfloat16, device="cuda"), kl_layers=kl,
                         vl_layers=kl, local_base=dev(np.zeros((1,), np.int32)), W=W)
    assert e.value.code == 2
