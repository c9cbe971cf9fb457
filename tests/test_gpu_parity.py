"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Index lists must be bit-exact; attention outputs within 3e-3 (max abs) of the
fp64 oracle and lse within 1e-3. Sizes span several tiles, ragged tails,
adversarial ties and the degenerate cases (W = 0, k = 1, early positions)."""
import numpy as np
import pytest
import torch

import synth
from oracle import csa2_oracle as O
from oracle.workload import OracleCache, run_units
from sparse_attention_shared_b200 import ops

from gpu_util import (DeviceWorkload, assert_attn_close, assert_list_invariants, assert_lists_equal, bf16_dev,
                      dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ws():
    return ops.Workspace()


@pytest.fixture
def status():
    s = ops.Status()
    yield s
    s.check("after test")


# ---------------------------------------------------------------- FP4 codec
def test_fp4_quantize_bit_exact():
    x = synth.normal_f32(0, 77, (4096, 128))
    rng = np.random.default_rng(0)
    special = np.zeros((8, 128), np.float32)
    special[1] = 1e-6                                      # scale rounds to zero
    special[2] = rng.standard_normal(128) * 1000           # saturating scale
    e4 = torch.arange(1, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for r in range(3, 8):                                   # grid values and exact E2M1 midpoints
        s = e4[rng.integers(0, len(e4), 8)].repeat(16)
        m = np.array([0, .25, .5, .75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, -6], np.float32)
        special[r] = (m[rng.integers(0, 16, 128)] * s * rng.choice([-1, 1], 128)).astype(np.float32)
        special[r, ::16] = 6 * s[::16]
    x = np.concatenate([x, special])
    codes, scales = ops.fp4_quantize(dev(x))
    rc, rs = O.fp4_quantize(x)
    assert_lists_equal(scales, rs, "scales")
    assert_lists_equal(codes, rc, "codes")


# ---------------------------------------------------------------- indexer
def _oracle_full(qi, w, ki, q_pos, k, P):
    B, Tq = q_pos.shape
    pools = np.full((B, Tq, max(P, 1)), -1, np.int32)
    topk = np.full((B, Tq, k), -1, np.int32)
    for b in range(B):
        for j in range(Tq):
            p, t = O.index_full(qi[b, j], w, ki[b], int(q_pos[b, j]), k, P)
            topk[b, j] = t
            if P:
                pools[b, j] = p
    return (pools if P else None), topk


def _check_full(qi, w, ki, q_pos, k, P, ws, status):
    pool, topk = ops.index_topk("FULL", dev(q_pos), dev(qi), w, dev(ki), k, P, ws=ws, status=status)
    rpool, rtopk = _oracle_full(qi, w, ki, q_pos, k, P)
    assert_list_invariants(topk.cpu().numpy(), q_pos, "topk")
    assert_lists_equal(topk, rtopk, "topk")
    if P:
        assert_list_invariants(pool.cpu().numpy(), q_pos, "pool")
        assert_lists_equal(pool, rpool, "pool")
    return pool, topk


def test_index_full_tiny(ws, status):
    wl = synth.make_workload("tiny")
    for P in (0, 512):
        _check_full(wl.qi(0), wl.w(0), wl.ki(0), wl.q_pos(), 256, P, ws, status)


@pytest.mark.parametrize("B,N,Tq,k,P", [(4, 8192, 1, 2048, 4096), (3, 5000, 2, 300, 1000), (2, 20000, 1, 2048, 8192),
                                        (1, 70001, 1, 2048, 8192), (40, 3000, 1, 100, 0),
                                        # more units than SMs: one CTA per unit, scores spilled past 16384
                                        (150, 20000, 1, 512, 2048)])
def test_index_full_shapes(B, N, Tq, k, P, ws, status):
    qi = synth.randint_i8(1, 10 + B, (B, Tq, 8, 64))
    ki = synth.randint_i8(1, 20 + N, (B, N, 64))
    w = synth.randint_i32(1, 30, (8,), 1, 8)
    q_pos = np.broadcast_to(np.arange(N - Tq, N, dtype=np.int32), (B, Tq)).copy()
    _check_full(qi, w, ki, q_pos, k, P, ws, status)


@pytest.mark.parametrize("B,N,Tq,Hi,Di,k,P", [
    (2, 9000, 20, 8, 64, 300, 1000),     # blocks of 16 + 4 queries, positions spread over the second half
    (1, 8192, 5, 6, 128, 100, 0),        # 128-byte keys, 6 heads
    (3, 20000, 40, 8, 64, 2048, 8192),   # scores past 16384 per CTA
    (1, 12000, 16, 4, 32, 256, 512),     # 32-byte keys, 4 heads
])
def test_index_full_shared_keys(B, N, Tq, Hi, Di, k, P, ws, status):
    """Tq >= 4 queries per sequence: blocks of queries share key tiles; sampled tiles give
    each query a threshold estimate, the marking pass records its candidates, and one CTA
    per query rescores and cuts them (a query with fewer positions than k takes them all)."""
    qi = synth.randint_i8(3, 10 + Tq, (B, Tq, Hi, Di))
    ki = synth.randint_i8(3, 20 + N, (B, N, Di))
    w = synth.randint_i32(3, 30, (Hi,), 1, 8)
    rng = np.random.default_rng(N + Tq)
    q_pos = np.sort(rng.integers(N // 2, N, size=(B, Tq)), axis=1).astype(np.int32)
    q_pos[:, -1] = N - 1
    q_pos[0, 0] = min(q_pos[0, 0], 5)        # a query with fewer positions than k
    _check_full(qi, w, ki, q_pos, k, P, ws, status)


def test_index_shared_keys_bad_positions(ws):
    """A shared-key call with positions outside [0, N): the status word says
    CSA2_ERR_RANGE, those queries' lists are all -1, and every other query's lists are
    exact."""
    B, N, Tq, Hi, Di, k, P = 1, 9000, 20, 8, 64, 300, 1000
    qi = synth.randint_i8(5, 1, (B, Tq, Hi, Di))
    ki = synth.randint_i8(5, 2, (B, N, Di))
    w = synth.randint_i32(5, 3, (Hi,), 1, 8)
    q_pos = np.sort(np.random.default_rng(7).integers(N // 2, N, size=(B, Tq)), axis=1).astype(np.int32)
    bad = [3, 11]
    q_pos[0, 3], q_pos[0, 11] = -1, N
    st = ops.Status()
    pool, topk = ops.index_topk("FULL", dev(q_pos), dev(qi), w, dev(ki), k, P, ws=ws, status=st)
    code, _ = st.read()
    assert code == 5   # CSA2_ERR_RANGE
    good = [j for j in range(Tq) if j not in bad]
    rpool, rtopk = _oracle_full(qi[:, good], w, ki, q_pos[:, good], k, P)
    got_t, got_p = topk.cpu().numpy(), pool.cpu().numpy()
    assert_lists_equal(torch.from_numpy(np.ascontiguousarray(got_t[:, good])), rtopk, "topk")
    assert_lists_equal(torch.from_numpy(np.ascontiguousarray(got_p[:, good])), rpool, "pool")
    assert (got_t[:, bad] == -1).all() and (got_p[:, bad] == -1).all()


def test_index_full_early_positions_and_padding(ws, status):
    B, N = 2, 4096
    qi = synth.randint_i8(2, 1, (B, 6, 8, 64))
    ki = synth.randint_i8(2, 2, (B, N, 64))
    w = synth.randint_i32(2, 3, (8,), 1, 8)
    q_pos = np.array([[0, 1, 100, 300, 2047, 4095], [5, 255, 256, 257, 1000, 3000]], np.int32)
    _check_full(qi, w, ki, q_pos, 300, 600, ws, status)


@pytest.mark.parametrize("kind", ["all_equal", "relu_zero", "half_equal", "negative_w", "few_values"])
def test_index_ties(kind, ws, status):
    B, N, Tq = 2, 30000, 1
    rng = np.random.default_rng(5)
    qi = synth.randint_i8(3, 1, (B, Tq, 8, 64))
    ki = synth.randint_i8(3, 2, (B, N, 64))
    w = synth.randint_i32(3, 3, (8,), 1, 8)
    if kind == "all_equal":
        ki[:] = 5
    elif kind == "relu_zero":
        qi[:] = 100
        ki[:] = -127
    elif kind == "half_equal":
        ki[:, ::2] = 7
    elif kind == "negative_w":
        w = -w
    elif kind == "few_values":
        ki[:] = rng.integers(-2, 3, ki.shape).astype(np.int8)
        qi[:] = 1
    q_pos = np.full((B, Tq), N - 1, np.int32)
    _check_full(qi, w, ki, q_pos, 2048, 8192, ws, status)


@pytest.mark.parametrize("where", ["front", "back"])
def test_index_full_concentrated_top(where, ws, status):
    """Keys aligned with the weighted index query in ~9000 neighbouring positions:
    one CTA's chunk then holds nearly all of the top-8192, so its warps' ordered
    lists overflow and the write falls back to the pass over the whole chunk."""
    B, N, A = 16, 131072, 9000
    qi = synth.randint_i8(7, 1, (B, 1, 8, 64))
    ki = synth.randint_i8(7, 2, (B, N, 64))
    w = synth.randint_i32(7, 3, (8,), 1, 8)
    noise = synth.randint_i32(7, 4, (B, A, 64), -37, 37)
    for b in range(B):
        v = (w[:, None].astype(np.int64) * qi[b, 0].astype(np.int64)).sum(0)
        rows = slice(0, A) if where == "front" else slice(N - A, N)
        ki[b, rows] = np.clip(np.sign(v)[None, :] * 90 + noise[b], -127, 127).astype(np.int8)
    q_pos = np.full((B, 1), N - 1, np.int32)
    _check_full(qi, w, ki, q_pos, 2048, 8192, ws, status)


def test_index_sequence_shares_workspace(ws, status):
    """Full, Full, Reindex (one select per group), Full on one workspace. The
    indexer keeps three rotating level-0 histogram buffers per group; every kernel
    must leave the next one zero whichever select it ran, or the last Full call
    reads the histogram the first one left behind."""
    B, N = 16, 65536
    qs = [synth.randint_i8(8, i, (B, 1, 8, 64)) for i in range(4)]
    ki = synth.randint_i8(8, 10, (B, N, 64))
    w = synth.randint_i32(8, 11, (8,), 1, 8)
    q_pos = np.full((B, 1), N - 1, np.int32)
    _check_full(qs[0], w, ki, q_pos, 2048, 8192, ws, status)
    pool, _ = _check_full(qs[1], w, ki, q_pos, 2048, 8192, ws, status)
    _, t2 = ops.index_topk("REINDEX", dev(q_pos), dev(qs[2]), w, dev(ki), 2048, pool_in=pool, ws=ws, status=status)
    rp = pool.cpu().numpy()
    ref = np.stack([[O.index_reindex(qs[2][b, 0], w, ki[b], rp[b, 0], 2048)] for b in range(B)])
    assert_lists_equal(t2, ref, "reindex topk")
    _check_full(qs[3], w, ki, q_pos, 2048, 8192, ws, status)


def test_index_reindex(ws, status):
    B, N = 3, 12000
    qi = synth.randint_i8(4, 1, (B, 1, 8, 64))
    ki = synth.randint_i8(4, 2, (B, N, 64))
    w = synth.randint_i32(4, 3, (8,), 1, 8)
    q_pos = np.array([[N - 1], [N - 1], [3000]], np.int32)
    pool, _ = _check_full(qi, w, ki, q_pos, 1024, 4096, ws, status)
    qi2 = synth.randint_i8(4, 4, (B, 1, 8, 64))
    ki2 = synth.randint_i8(4, 5, (B, N, 64))
    w2 = synth.randint_i32(4, 6, (8,), 1, 8)
    _, topk2 = ops.index_topk("REINDEX", dev(q_pos), dev(qi2), w2, dev(ki2), 1024, pool_in=pool, ws=ws, status=status)
    rpool = pool.cpu().numpy()
    ref = np.stack([[O.index_reindex(qi2[b, 0], w2, ki2[b], rpool[b, 0], 1024)] for b in range(B)])
    assert_lists_equal(topk2, ref, "reindex topk")
    for b in range(B):
        got = set(topk2[b, 0].cpu().numpy().tolist()) - {-1}
        assert got <= set(rpool[b, 0].tolist())


def test_index_reindex_concentrated_top(ws, status):
    """A 16384-entry pool whose keys are aligned with the weighted index query in one
    band of positions: the group's single select finds the whole top-k in a few warps'
    ranges, their ordered lists overflow, and the cut falls back to the passes over
    all scores."""
    B, N, P, k = 16, 40000, 16384, 2048
    qi = synth.randint_i8(9, 1, (B, 1, 8, 64))
    ki = synth.randint_i8(9, 2, (B, N, 64))
    w = synth.randint_i32(9, 3, (8,), 1, 8)
    pool = np.broadcast_to(np.arange(P, dtype=np.int32), (B, 1, P)).copy()
    noise = synth.randint_i32(9, 4, (B, 3000, 64), -37, 37)
    for b in range(B):
        v = (w[:, None].astype(np.int64) * qi[b, 0].astype(np.int64)).sum(0)
        ki[b, 2000:5000] = np.clip(np.sign(v)[None, :] * 90 + noise[b], -127, 127).astype(np.int8)
    q_pos = np.full((B, 1), N - 1, np.int32)
    _, t2 = ops.index_topk("REINDEX", dev(q_pos), dev(qi), w, dev(ki), k, pool_in=dev(pool), ws=ws, status=status)
    ref = np.stack([[O.index_reindex(qi[b, 0], w, ki[b], pool[b, 0], k)] for b in range(B)])
    assert_lists_equal(t2, ref, "reindex topk")


def test_index_reindex_ties_small_pool(ws, status):
    B, N = 2, 5000
    qi = synth.randint_i8(6, 1, (B, 1, 4, 32))
    ki = np.full((B, N, 32), 3, np.int8)
    w = np.array([1, 2, 3, 4], np.int32)
    q_pos = np.array([[N - 1], [200]], np.int32)
    pool, _ = _check_full(qi, w, ki, q_pos, 100, 500, ws, status)
    _, t2 = ops.index_topk("REINDEX", dev(q_pos), dev(qi), w, dev(ki), 100, pool_in=pool, ws=ws, status=status)
    rp = pool.cpu().numpy()
    ref = np.stack([[O.index_reindex(qi[b, 0], w, ki[b], rp[b, 0], 100)] for b in range(B)])
    assert_lists_equal(t2, ref, "reindex ties")


# ---------------------------------------------------------------- attention
def _attn_case(B, N, Tq, Hq, D, k, W, seed, topk_fn=None, ws=None, status=None):
    kv = synth.normal_f32(seed, 1, (B, N, D))
    codes, scales = O.fp4_quantize(kv)
    q = synth.normal_bf16(seed, 2, (B, Tq, Hq, D))
    base = max(0, N - Tq - W + 1)
    Lloc = N - base
    kl = synth.normal_bf16(seed, 3, (B, max(Lloc, 1), D))
    vl = synth.normal_bf16(seed, 4, (B, max(Lloc, 1), D))
    q_pos = np.broadcast_to(np.arange(N - Tq, N, dtype=np.int32), (B, Tq)).copy()
    rng = np.random.default_rng(seed)
    topk = np.full((B, Tq, k), -1, np.int32)
    for b in range(B):
        for j in range(Tq):
            t = q_pos[b, j]
            sel = topk_fn(t, rng) if topk_fn else np.sort(rng.choice(t + 1, min(k, t + 1), replace=False))
            topk[b, j, :len(sel)] = sel
    gcodes, gscales = ops.fp4_quantize(dev(kv.reshape(-1, D)))
    out, lse = ops.sparse_attn(dev(q_pos), bf16_dev(q), gcodes.view(B, N, D // 2), gscales.view(B, N, D // 16),
                               dev(topk), bf16_dev(kl) if W else None, bf16_dev(vl) if W else None,
                               dev(np.full((B,), base, np.int32)) if W else None, W, ws=ws, status=status)
    ref_o = np.zeros((B, Tq, Hq, D))
    ref_l = np.zeros((B, Tq, Hq))
    for b in range(B):
        klf, vlf = O.bf16_to_f64(kl[b]), O.bf16_to_f64(vl[b])
        for j in range(Tq):
            ref_o[b, j], ref_l[b, j] = O.attention_unit(O.bf16_to_f64(q[b, j]), codes[b], scales[b], topk[b, j],
                                                       klf, vlf, base, int(q_pos[b, j]), W)
    return assert_attn_close(out, lse, ref_o, ref_l, f"attn B{B} N{N} Tq{Tq} Hq{Hq} D{D} k{k} W{W}")


def test_attention_tiny(ws, status):
    wl = synth.make_workload("tiny")
    dw = DeviceWorkload(wl)
    s = wl.spec
    _, topk = O.index_full(wl.qi(0)[0, 0], wl.w(0), wl.ki(0)[0], 2047, 256)
    topks = np.stack([[O.index_full(wl.qi(0)[0, j], wl.w(0), wl.ki(0)[0], int(wl.q_pos()[0, j]), 256)[1]
                       for j in range(s.Tq)]])
    out, lse = ops.sparse_attn(dw.q_pos, bf16_dev(wl.q(0)), dw.kv_fp4, dw.kv_scale, dev(topks), bf16_dev(wl.kl(0)),
                               bf16_dev(wl.vl(0)), dw.local_base, s.W, ws=ws, status=status)
    res = run_units(wl, [(0, j) for j in range(s.Tq)])
    ro = np.stack([[res[(0, j)][0]["out"] for j in range(s.Tq)]])
    rl = np.stack([[res[(0, j)][0]["lse"] for j in range(s.Tq)]])
    assert_lists_equal(dev(topks), np.stack([[res[(0, j)][0]["topk"] for j in range(s.Tq)]]), "oracle topk")
    assert_attn_close(out, lse, ro, rl, "tiny attention")


@pytest.mark.parametrize("B,N,Tq,Hq,D,k,W", [
    (2, 4096, 1, 16, 128, 2048, 512),
    (3, 3000, 2, 16, 128, 300, 200),     # ragged tiles on both branches
    (2, 2500, 3, 32, 128, 256, 128),     # 32 heads (prefill shape)
    (2, 2048, 2, 8, 64, 256, 128),       # D = 64, padded heads
    (2, 4096, 1, 16, 128, 1, 0),         # single global entry, no window
    (2, 4096, 1, 16, 128, 2048, 0),      # no local branch
    (1, 300, 1, 16, 128, 512, 64),       # fewer positions than k: -1 padding
    (2, 8192, 1, 16, 128, 4096, 1024),   # 16 list CTAs + 8 window CTAs: past the cluster limit, ticket merge
    (2, 8192, 1, 16, 128, 4096, 2048),   # 16 window tiles: ticket merge
    (3, 5000, 1, 32, 64, 700, 300),      # 32 heads at D = 64, ragged blocks
    (2, 4096, 1, 16, 128, 1, 512),       # one global entry, four window tiles
    (1, 20000, 1, 32, 128, 100, 16284),  # k + W = 16384 with both branches ragged: 129 tiles, 32 heads
    (1, 3000, 300, 32, 64, 700, 300),    # 300 queries: one CTA per query over all tiles, 32 heads, D = 64
    (1, 3000, 300, 8, 64, 256, 128),     # the same at 16 (padded) heads
    (2, 5000, 160, 16, 128, 1000, 200),  # 320 queries over two sequences, ragged tiles, D = 128
])
def test_attention_shapes(B, N, Tq, Hq, D, k, W, ws, status):
    _attn_case(B, N, Tq, Hq, D, k, W, seed=B * 7 + N, ws=ws, status=status)


def test_attention_overlap_window_and_global(ws, status):
    """Positions in both the list and the window are counted twice."""
    def sel(t, rng):
        return np.arange(t - 63, t + 1)           # the last 64 positions, all inside the window
    _attn_case(2, 2048, 1, 16, 128, 64, 128, seed=9, topk_fn=sel, ws=ws, status=status)


def test_attention_reports_bad_positions(ws):
    st = ops.Status()
    B, N, D = 1, 512, 128
    kv = synth.normal_f32(1, 1, (B * N, D))
    c, s = ops.fp4_quantize(dev(kv))
    topk = dev(np.array([[[0, 5, 700, -1]]], np.int32))      # 700 >= N
    ops.sparse_attn(dev(np.array([[N - 1]], np.int32)), bf16_dev(synth.normal_bf16(1, 2, (B, 1, 16, D))),
                    c.view(B, N, D // 2), s.view(B, N, D // 16), topk, None, None, None, 0, ws=ws, status=st)
    code, _ = st.read()
    assert code == 5   # CSA2_ERR_RANGE


# ---------------------------------------------------------------- layer stack
def _check_stack(wl, units, ws, status, keep_reuse=True):
    dw = DeviceWorkload(wl)
    st = ops.LayerStack(dw.layer_dicts(), dw.q_pos, dw.kv_fp4, dw.kv_scale, dw.local_base, keep_reuse_lists=keep_reuse)
    st.run(ws, status)
    torch.cuda.synchronize()
    res = run_units(wl, units)
    worst = 0.0
    for (b, j), layers in res.items():
        last_src = None
        for li, r in enumerate(layers):
            if st.topks[li] is not None:
                assert_lists_equal(st.topks[li][b, j], r["topk"], f"layer {li} ({r['mode']}) topk unit {(b, j)}")
            if st.pools[li] is not None:
                assert_lists_equal(st.pools[li][b, j], r["pool"], f"layer {li} pool unit {(b, j)}")
            if r["mode"] == "REUSE" and st.topks[li] is not None:
                assert torch.equal(st.topks[li][b, j], st.topks[last_src][b, j])
            if r["mode"] != "REUSE":
                last_src = li
            worst = max(worst, assert_attn_close(st.outs[li][b, j], st.lses[li][b, j], r["out"], r["lse"],
                                                 f"layer {li} unit {(b, j)}"))
    return worst


def test_layer_stack_stack20_schedule_small(ws, status):
    wl = synth.make_workload("stack20_128k", B=2, N=16384)
    _check_stack(wl, [(0, 0), (1, 0)], ws, status)


def test_layer_stack_long_schedule_small(ws, status):
    wl = synth.make_workload("long_1m", N=40000, Tq=8)
    _check_stack(wl, [(0, j) for j in range(8)], ws, status)


@pytest.mark.parametrize("keep_reuse", [True, False])
def test_layer_stack_paper_schedule_small(keep_reuse, ws, status):
    # keep_reuse=False: Reuse layers gather their global rows before the previous kernel ends
    wl = synth.make_workload("paper_schedule", B=3, N=9000)
    _check_stack(wl, [(b, 0) for b in range(3)], ws, status, keep_reuse=keep_reuse)


def test_layer_stack_rejects_bad_mode_order(ws):
    wl = synth.make_workload("stack20_128k", B=1, N=4096)
    dw = DeviceWorkload(wl)
    layers = dw.layer_dicts()
    with pytest.raises(ValueError):
        ops.LayerStack([layers[1]] + layers[1:], dw.q_pos, dw.kv_fp4, dw.kv_scale, dw.local_base)   # REUSE first
    with pytest.raises(ValueError):
        ops.LayerStack([layers[3]], dw.q_pos, dw.kv_fp4, dw.kv_scale, dw.local_base)                # REINDEX first


# ---------------------------------------------------------------- full-size workloads, every unit
def _check_stack_every_unit(wl, ws, status):
    """The whole workload through the CUDA stack; every query's pool and top-k list of
    every layer compared bit for bit with the C++ oracle (threads over units), every
    list checked for the causal layout, and every query's output and lse at every
    layer compared within the tolerances."""
    from oracle import cpp as C
    s = wl.spec
    dw = DeviceWorkload(wl)
    st = ops.LayerStack(dw.layer_dicts(), dw.q_pos, dw.kv_fp4, dw.kv_scale, dw.local_base, keep_reuse_lists=False,
                        m=s.m)
    st.run(ws, status)
    torch.cuda.synchronize()
    status.check("stack")
    q_pos = wl.q_pos()
    lists = C.stack_lists(wl)
    for li, e in enumerate(lists):
        if st.topks[li] is not None:
            assert_list_invariants(st.topks[li].cpu().numpy(), q_pos, f"layer {li} topk")
            assert_lists_equal(st.topks[li], e["topk"], f"layer {li} ({e['mode']}) topk, every unit")
        if st.pools[li] is not None:
            assert_list_invariants(st.pools[li].cpu().numpy(), q_pos, f"layer {li} pool")
            assert_lists_equal(st.pools[li], e["pool"], f"layer {li} pool, every unit")
    kv = wl.kv_f32() if s.m <= 1 else C.compress_entries(wl.kv_f32(), s.m)
    codes, scales = C.fp4_quantize(kv)
    assert_lists_equal(dw.kv_fp4, codes, "FP4 codes of the cache")
    assert_lists_equal(dw.kv_scale, scales, "E4M3 scales of the cache")
    outs = C.stack_outputs(wl, codes, scales, lists, range(s.B))
    worst = 0.0
    for li in range(s.L):
        worst = max(worst, assert_attn_close(st.outs[li], st.lses[li], outs[li]["out"], outs[li]["lse"],
                                             f"layer {li}, every unit"))
    return worst


def test_decode_full_every_unit(ws, status):
    _check_stack_every_unit(synth.make_workload("decode_full"), ws, status)


def test_prefill_chunk_every_unit(ws, status):
    # 4096 queries of one sequence, 32 heads: the shared-key Full path (sampled estimates, candidate bits, the
    # tensor-core cut at two queries per SM) and the per-query attention
    _check_stack_every_unit(synth.make_workload("prefill_chunk"), ws, status)


def test_long_1m_every_unit(ws, status):
    # one sequence of 2^20 positions, 64 queries: the shared-key Full path (128 sampled tiles a query, the
    # one-CTA cut), nine Reindex layers select from the pool by the group's single select
    _check_stack_every_unit(synth.make_workload("long_1m"), ws, status)


def test_stack20_128k_every_unit(ws, status):
    _check_stack_every_unit(synth.make_workload("stack20_128k"), ws, status)


def test_paper_schedule_every_unit(ws, status):
    # the pages' own schedule at full size: [Full + 3 Reuse] + 4 x [Reindex + 3 Reuse] on one shared key set,
    # pool 2048 and top-512 (the Reindex groups take four CTAs of 512 pool entries a query), SWA 128
    _check_stack_every_unit(synth.make_workload("paper_schedule"), ws, status)


def test_encoder_m2_shared_keys_every_unit(ws, status):
    # compression rate 2 with 8 queries a sequence: the shared-key Full path reads entries up to each
    # query's last one ((t + 1) / 2 - 1), then Reuse and Reindex layers
    _check_stack_every_unit(synth.make_workload("encoder_m2", B=2, N=20000, Tq=8), ws, status)


def test_tiny_every_unit(ws, status):
    _check_stack_every_unit(synth.make_workload("tiny"), ws, status)


def test_replay_prefill_every_unit(ws, status):
    # bounded replay: the last 256 of 16384 prompt positions through [F,U,U,RI]x5, window references cut at
    # the segment (local_base = N - 256); the Full layers take the shared-key path, the Reindex layers the
    # tensor-core cut over the pool (512 queries, more than SMs)
    wl = synth.make_workload("replay_prefill", B=2, N=16384, Tq=256, W=256)
    assert wl.spec.local_base == 16384 - 256
    _check_stack_every_unit(wl, ws, status)


def test_encoder_m2_every_unit(ws, status):
    # sequence compression rate 2: 4096 entries (each the mean of two positions) for 8192 positions; queries
    # at an odd and an even position read only complete entries
    wl = synth.make_workload("encoder_m2", B=3, N=4096, Tq=2)
    assert wl.spec.n_pos == 8192
    _check_stack_every_unit(wl, ws, status)


def test_encoder_m2_early_positions(ws, status):
    """Queries at positions 0..5 with m = 2 read entries 0..(t+1)/2-1: none at t = 0."""
    B, Nent, m = 1, 64, 2
    qi = synth.randint_i8(12, 1, (B, 6, 8, 64))
    ki = synth.randint_i8(12, 2, (B, Nent, 64))
    w = synth.randint_i32(12, 3, (8,), 1, 8)
    q_pos = np.arange(6, dtype=np.int32)[None, :]
    _, topk = ops.index_topk("FULL", dev(q_pos), dev(qi), w, dev(ki), 4, ws=ws, status=status, m=m)
    got = topk.cpu().numpy()
    for j in range(6):
        _, ref = O.index_full(qi[0, j], w, ki[0], j, 4, 0, m)
        assert np.array_equal(got[0, j], ref)
        assert (got[0, j] >= 0).sum() == min(4, (j + 1) // 2)


def test_one_workspace_serves_calls_of_different_sizes(status):
    """A workspace is zeroed once and then serves calls of any sizes in turn. A Full call
    over 4 queries that share 2^20 keys leaves their scores in its scratch; an attention
    call over 320 queries that then merges by tickets (one CTA per tile) must find its
    tickets zero, so the ticket region may not move with the number of queries."""
    ws = ops.Workspace()
    N1 = 1 << 20
    qi = synth.randint_i8(5, 1, (1, 4, 8, 64))
    ki = synth.randint_i8(5, 2, (1, N1, 64))
    w = synth.randint_i32(5, 3, (8,), 1, 8)
    q_pos = np.arange(N1 - 4, N1, dtype=np.int32)[None, :]
    ops.index_topk("FULL", dev(q_pos), dev(qi), w, dev(ki), 2048, 0, ws=ws, status=status)
    status.check("Full call")
    _attn_case(1, 4096, 320, 16, 128, 256, 128, seed=9, ws=ws, status=status)
