"""Pins of the plain C++17 oracle (oracle/csa2_oracle.cpp).

Each of its functions is checked against something other than itself: the
published format tables (torch's float8 cast, the OCP E2M1 values and tie rule),
brute force in plain Python integers, the pages' worked examples (Fig. 4, Fig. 5
of "CED: Continuing Context with a Causal Encoder and Decoder"), closed forms of
attention (one entry, dense equivalence against torch's fp64 SDPA) and the
independent numpy oracle, which it must match bit for bit on lists and codes and
to 1e-12 on attention outputs."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import cpp as C
from oracle import csa2_oracle as O
from oracle.workload import OracleCache, run_units


# ---------------------------------------------------------------- formats
def test_e4m3_values_match_torch_cast():
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([C.lib().orc_e4m3_value(b) for b in range(256)])
    fin = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[fin], ref[fin])


def test_e2m1_values_match_published_table(golden):
    g = golden("e2m1_values.json")
    got = [C.lib().orc_e2m1_value(c) for c in range(16)]
    assert got == [float(v) for v in g["values"]]


def test_e2m1_ties_golden(golden):
    g = golden("e2m1_rne_ties.json")
    got = [C.lib().orc_e2m1_value(C.lib().orc_e2m1_round(x)) for x in g["inputs"]]
    assert got == [float(v) for v in g["expected"]]


def test_e4m3_round_matches_torch_cast():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(-14, 6, 3000))])
    pos = torch.arange(127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = (pos[1:] + pos[:-1]) / 2                       # every midpoint: ties to even
    vals = np.concatenate([vals, mids])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([C.lib().orc_e4m3_round(float(v)) for v in vals])
    assert np.array_equal(got, ref)
    assert C.lib().orc_e4m3_round(1e6) == 0x7E           # saturates at 448


def test_fp4_quantize_matches_numpy_oracle_bit_exact():
    x = synth.normal_f32(3, 9, (512, 128))
    rng = np.random.default_rng(2)
    special = np.zeros((6, 128), np.float32)
    special[1] = 1e-6
    special[2] = rng.standard_normal(128) * 1000
    grid = np.array([0, .25, .5, .75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, -6], np.float32)
    for r in range(3, 6):
        special[r] = grid[rng.integers(0, 16, 128)] * np.float32(0.375)
        special[r, ::16] = 6 * np.float32(0.375)
    x = np.concatenate([x, special])
    c1, s1 = C.fp4_quantize(x)
    c2, s2 = O.fp4_quantize(x)
    assert np.array_equal(s1, s2) and np.array_equal(c1, c2)


def test_fp4_value_every_code_and_scale():
    L = C.lib()
    codes = np.zeros(1, np.uint8)
    scales = np.zeros(1, np.uint8)
    for sc in range(256):
        scales[0] = sc
        for c in range(16):
            codes[0] = c
            v = L.orc_fp4_value(codes.ctypes.data, scales.ctypes.data, 0)
            ref = O.e2m1_value(c) * O.e4m3_value(sc)
            assert (math.isnan(v) and math.isnan(ref)) or v == ref


def test_roundtrip_exact_on_grid_blocks():
    rng = np.random.default_rng(4)
    s = O.e4m3_value(np.arange(1, 100))
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    x = np.zeros((64, 32), np.float32)
    for r in range(64):
        for g in range(2):
            sc = s[rng.integers(0, len(s))]
            blk = grid[rng.integers(0, 8, 16)] * rng.choice([-1, 1], 16)
            blk[rng.integers(0, 16)] = 6
            x[r, 16 * g:16 * g + 16] = (blk * sc).astype(np.float32)
    codes, scales = C.fp4_quantize(x)
    assert np.array_equal(O.fp4_dequantize(codes, scales), x.astype(np.float64))


# ---------------------------------------------------------------- indexer
def _py_full(qi, w, keys, t, count):
    sc = []
    for s in range(min(t, len(keys) - 1) + 1):
        tot = 0
        for h in range(len(qi)):
            tot += int(w[h]) * max(0, sum(int(a) * int(b) for a, b in zip(qi[h], keys[s])))
        sc.append((tot, s))
    sc.sort(key=lambda x: (-x[0], x[1]))
    sel = sorted(s for _, s in sc[:count])
    return sel + [-1] * (count - len(sel))


@pytest.mark.parametrize("seed", range(3))
def test_full_bruteforce_every_k(seed):
    rng = np.random.default_rng(300 + seed)
    N, Hi, Di = 40, 3, 16
    keys = rng.integers(-128, 128, (N, Di)).astype(np.int8)
    keys[::5] = keys[1]                                   # ties
    qi = rng.integers(-128, 128, (Hi, Di)).astype(np.int8)
    w = rng.integers(-3, 9, Hi).astype(np.int32)
    for t in (0, 7, N - 1):
        for k in (1, 2, 5, 17, 41, 50):
            _, topk = C.index_full(qi, w, keys, t, k)
            assert topk.tolist() == _py_full(qi, w, keys, t, k)


def test_fig4_selection(golden):
    g = golden("fig4_selection.json")
    _, topk = C.index_full(np.array(g["qi"]), np.array(g["w"]), np.array(g["keys"]), g["t"], g["k"])
    assert topk.tolist() == g["expected_topk"]


def test_fig5_full_reindex_reuse(golden):
    g = golden("fig5_modes.json")
    f, r = g["full"], g["reindex"]
    pool, topk = C.index_full(np.array(f["qi"]), np.array(f["w"]), np.array(f["keys"]), g["t"], g["k"], g["P"])
    assert pool.tolist() == g["expected_full_pool"] and topk.tolist() == g["expected_full_topk"]
    t2 = C.index_reindex(np.array(r["qi"]), np.array(r["w"]), np.array(r["keys"]), pool, g["k"])
    assert t2.tolist() == g["expected_reindex_topk"]
    assert t2.tolist() == g["expected_reuse_topk"]        # Reuse reads the list unchanged


def test_full_and_reindex_match_numpy_oracle():
    rng = np.random.default_rng(7)
    N = 3000
    keys = synth.randint_i8(7, 1, (N, 64), -128, 127)
    for i in range(4):
        qi = synth.randint_i8(7, 2 + i, (8, 64), -128, 127)
        w = rng.integers(1, 9, 8).astype(np.int32)
        t = int(rng.integers(100, N))
        p1, t1 = C.index_full(qi, w, keys, t, 256, 700)
        p2, t2 = O.index_full(qi, w, keys, t, 256, 700)
        assert np.array_equal(p1, p2) and np.array_equal(t1, t2)
        r1 = C.index_reindex(qi[::-1].copy(), w, keys, p1, 200)
        assert np.array_equal(r1, O.index_reindex(qi[::-1].copy(), w, keys, p1, 200))
        assert set(r1.tolist()) - {-1} <= set(p1.tolist())


def test_reindex_over_full_pool_with_same_inputs_equals_full():
    keys = synth.randint_i8(8, 1, (500, 32))
    qi = synth.randint_i8(8, 2, (4, 32))
    w = np.array([1, 2, 3, 4], np.int32)
    pool, topk = C.index_full(qi, w, keys, 499, 50, 500)
    assert np.array_equal(C.index_reindex(qi, w, keys, pool, 50), topk)


def test_batched_index_matches_single_units():
    B, Tq, N = 3, 5, 2000
    qi = synth.randint_i8(9, 1, (B, Tq, 8, 64))
    ki = synth.randint_i8(9, 2, (B, N, 64))
    w = synth.randint_i32(9, 3, (8,), 1, 8)
    q_pos = np.sort(np.random.default_rng(9).integers(0, N, (B, Tq)), axis=1).astype(np.int32)
    pool, topk = C.index_full_batch(q_pos, qi, w, ki, 100, 300, threads=4)
    r = C.index_reindex_batch(qi, w, ki, pool, 60, threads=4)
    for b in range(B):
        for j in range(Tq):
            p1, t1 = O.index_full(qi[b, j], w, ki[b], int(q_pos[b, j]), 100, 300)
            assert np.array_equal(pool[b, j], p1) and np.array_equal(topk[b, j], t1)
            assert np.array_equal(r[b, j], O.index_reindex(qi[b, j], w, ki[b], p1, 60))


# ---------------------------------------------------------------- attention
def _bits(x):
    return (torch.from_numpy(np.asarray(x, np.float32)).bfloat16().view(torch.int16).numpy().view(np.uint16))


def test_single_entry_no_window_is_its_value():
    D = 64
    x = synth.normal_f32(5, 1, (10, D))
    codes, scales = C.fp4_quantize(x)
    q = _bits(synth.normal_f32(5, 2, (4, D)))
    topk = np.array([6, -1, -1], np.int32)
    out, lse = C.attention_unit(q, codes, scales, topk, None, None, 0, 9, 0)
    g = O.fp4_dequantize(codes[6], scales[6])
    assert np.array_equal(out, np.broadcast_to(g, out.shape))
    qf = O.bf16_to_f64(q)
    assert np.allclose(lse, qf @ g / math.sqrt(D), rtol=0, atol=1e-12)


def test_dense_equivalence_against_sdpa():
    """Top-k over the whole causal prefix with W = 0 is dense causal attention over
    the dequantised rows; with a window, attention over the explicit concatenation."""
    N, Hq, D, t, W, base = 300, 4, 64, 250, 40, 200
    x = synth.normal_f32(6, 1, (N, D))
    codes, scales = C.fp4_quantize(x)
    g = O.fp4_dequantize(codes, scales)
    q = _bits(synth.normal_f32(6, 2, (Hq, D)))
    kl = _bits(synth.normal_f32(6, 3, (N - base, D)))
    vl = _bits(synth.normal_f32(6, 4, (N - base, D)))
    qf = torch.from_numpy(O.bf16_to_f64(q))
    topk = np.arange(t + 1, dtype=np.int32)
    out, _ = C.attention_unit(q, codes, scales, topk, None, None, 0, t, 0)
    G = torch.from_numpy(g[: t + 1])
    ref = torch.nn.functional.scaled_dot_product_attention(qf[None], G[None], G[None])[0].numpy()
    assert np.abs(out - ref).max() < 1e-12
    out2, _ = C.attention_unit(q, codes, scales, topk, kl, vl, base, t, W)
    win = np.arange(max(base, t - W + 1), t + 1) - base
    K = torch.cat([G, torch.from_numpy(O.bf16_to_f64(kl)[win])])
    V = torch.cat([G, torch.from_numpy(O.bf16_to_f64(vl)[win])])
    ref2 = torch.nn.functional.scaled_dot_product_attention(qf[None], K[None], V[None])[0].numpy()
    assert np.abs(out2 - ref2).max() < 1e-12


def test_empty_union():
    out, lse = C.attention_unit(np.zeros((2, 64), np.uint16), np.zeros((4, 32), np.uint8),
                                np.zeros((4, 4), np.uint8), np.array([-1, -1], np.int32), None, None, 0, 3, 0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("name,kw,units", [
    ("stack20_128k", dict(B=2, N=5000), [(0, 0), (1, 0)]),
    ("long_1m", dict(N=6000, Tq=4), [(0, 0), (0, 3)]),
    ("paper_schedule", dict(B=2, N=3000), [(0, 0), (1, 0)]),
    ("tiny", {}, [(0, 0), (0, 15)]),
    ("decode_full", dict(B=3, N=4000), [(0, 0), (2, 0)]),
    ("prefill_chunk", dict(N=3000, Tq=40), [(0, 0), (0, 21), (0, 39)]),
    ("replay_prefill", dict(B=2, N=3000, Tq=64, W=64), [(0, 0), (1, 63)]),
    ("encoder_m2", dict(B=2, N=2000), [(0, 0), (1, 0)]),
])
def test_stack_matches_numpy_oracle(name, kw, units):
    """Lists bit-exact and outputs within 1e-12 of the numpy oracle through whole
    layer stacks (Full, Reindex over the most recent Full pool, Reuse)."""
    wl = synth.make_workload(name, **kw)
    lists = C.stack_lists(wl, threads=4)
    cache = OracleCache(wl)
    s = wl.spec
    seqs = sorted({b for b, _ in units})
    codes = np.stack([cache.seq(b)[0] if b in seqs else np.zeros_like(cache.seq(seqs[0])[0]) for b in range(s.B)])
    scales = np.stack([cache.seq(b)[1] if b in seqs else np.zeros_like(cache.seq(seqs[0])[1]) for b in range(s.B)])
    outs = C.stack_outputs(wl, codes, scales, lists, range(s.B), threads=4)
    ref = run_units(wl, units, cache)
    for (b, j), layers in ref.items():
        for li, r in enumerate(layers):
            assert np.array_equal(lists[li]["topk"][b, j], r["topk"]), (li, b, j)
            if r["pool"] is not None:
                assert np.array_equal(lists[li]["pool"][b, j], r["pool"])
            assert np.abs(outs[li]["out"][b, j] - r["out"]).max() < 1e-12
            assert np.abs(outs[li]["lse"][b, j] - r["lse"]).max() < 1e-12


@pytest.mark.parametrize("seed", range(12))
def test_random_small_calls_match_numpy_oracle(seed):
    """Random small shapes (head counts, widths, k, P, positions, windows, compression rate)."""
    rng = np.random.default_rng(1000 + seed)
    N = int(rng.integers(1, 400))
    Hi, Di = int(rng.integers(1, 17)), int(rng.choice([16, 32, 48, 64]))
    m = int(rng.choice([1, 1, 2]))
    keys = synth.randint_i8(seed, 1, (N, Di), -128, 127)
    if seed % 3 == 0:
        keys[:] = keys[0]                                   # all scores equal
    qi = synth.randint_i8(seed, 2, (Hi, Di), -128, 127)
    w = rng.integers(-5, 9, Hi).astype(np.int32)
    t = int(rng.integers(0, m * N))
    k = int(rng.integers(1, N + 3))
    P = int(rng.choice([0, k, k + int(rng.integers(0, 50))]))
    te = O.last_entry(t, m)
    p1, t1 = C.index_full(qi, w, keys, te, k, P)
    p2, t2 = O.index_full(qi, w, keys, t, k, P, m)
    assert np.array_equal(t1, t2)
    if P:
        assert np.array_equal(p1, p2)
        k2 = int(rng.integers(1, P + 1))
        assert np.array_equal(C.index_reindex(qi[::-1].copy(), w, keys, p1, k2),
                              O.index_reindex(qi[::-1].copy(), w, keys, p1, k2))
    D, Hq = int(rng.choice([64, 128])), int(rng.integers(1, 33))
    W = int(rng.integers(0, 40))
    npos = m * N
    base = max(0, t - W + 1 - int(rng.integers(0, 5)))
    x = synth.normal_f32(seed, 3, (N, D))
    codes, scales = C.fp4_quantize(x)
    q = _bits(synth.normal_f32(seed, 4, (Hq, D)))
    kl = _bits(synth.normal_f32(seed, 5, (max(1, npos - base), D)))
    vl = _bits(synth.normal_f32(seed, 6, (max(1, npos - base), D)))
    o1, l1 = C.attention_unit(q, codes, scales, t1, kl, vl, base, t, W)
    o2, l2 = O.attention_unit(O.bf16_to_f64(q), codes, scales, t1, O.bf16_to_f64(kl), O.bf16_to_f64(vl), base, t, W)
    fin = np.isfinite(l2)
    assert np.array_equal(np.isfinite(l1), fin)
    assert np.abs(o1 - o2).max() < 1e-12 and np.abs(l1[fin] - l2[fin]).max(initial=0) < 1e-12
