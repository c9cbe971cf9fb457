"""Pins of the oracle's attention against a library routine (torch scaled-dot-product
attention in fp64), the log-sum-exp merge identity, closed forms (k=1, q=0 averages) and
the union / overlap reading of Fig. 4."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import csa2_oracle as O


def _sdpa(q, k, v, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(k)[None, None].expand(1, q.shape[0], -1, -1),
        torch.from_numpy(v)[None, None].expand(1, q.shape[0], -1, -1), scale=scale)
    return out[0, :, 0, :].numpy()


def test_dense_equivalence_fp4_off_no_window():
    """k >= |prefix|, fp64 global values, W = 0: equals causal softmax attention."""
    rng = np.random.default_rng(0)
    N, D, Hq, t = 300, 64, 4, 250
    g = rng.standard_normal((N, D))
    q = rng.standard_normal((Hq, D))
    keys = rng.integers(-127, 128, (N, 16)).astype(np.int8)
    _, topk = O.index_full(rng.integers(-127, 128, (2, 16)).astype(np.int8), np.array([1, 2]), keys, t, N, 0)
    sel = topk[topk >= 0]
    assert sel.tolist() == list(range(t + 1))
    out, lse = O.attend(q, g[sel], g[sel], 1 / math.sqrt(D))
    ref = _sdpa(q, g[: t + 1], g[: t + 1], 1 / math.sqrt(D))
    assert np.abs(out - ref).max() < 1e-12
    lse_ref = torch.logsumexp(torch.from_numpy(q @ g[: t + 1].T / math.sqrt(D)), dim=1).numpy()
    assert np.abs(lse - lse_ref).max() < 1e-12


def test_dense_equivalence_with_window():
    rng = np.random.default_rng(1)
    N, D, Hq, t, W, base = 200, 32, 3, 180, 16, 150
    g = rng.standard_normal((N, D))
    kl = rng.standard_normal((N - base, D))
    vl = rng.standard_normal((N - base, D))
    q = rng.standard_normal((Hq, D))
    sel = np.arange(t + 1)
    win = O.window_positions(t, W, base) - base
    out, _ = O.attend(q, np.concatenate([g[sel], kl[win]]), np.concatenate([g[sel], vl[win]]), 0.2)
    ref = _sdpa(q, np.concatenate([g[: t + 1], kl[t - W + 1 - base: t + 1 - base]]),
                np.concatenate([g[: t + 1], vl[t - W + 1 - base: t + 1 - base]]), 0.2)
    assert np.abs(out - ref).max() < 1e-12


def test_lse_merge_identity():
    """Softmax over the union == log-sum-exp merge of the two branches."""
    rng = np.random.default_rng(2)
    q = rng.standard_normal((8, 64)) * 3
    a = rng.standard_normal((40, 64))
    kb, vb = rng.standard_normal((25, 64)), rng.standard_normal((25, 64))
    s = 1 / 8
    oa, la = O.attend(q, a, a, s)
    ob, lb = O.attend(q, kb, vb, s)
    ou, lu = O.attend(q, np.concatenate([a, kb]), np.concatenate([a, vb]), s)
    m = np.maximum(la, lb)
    wa, wb = np.exp(la - m), np.exp(lb - m)
    merged = (wa[:, None] * oa + wb[:, None] * ob) / (wa + wb)[:, None]
    assert np.abs(merged - ou).max() < 1e-12
    assert np.abs(m + np.log(wa + wb) - lu).max() < 1e-12


def test_single_global_entry_no_window_returns_its_value():
    wl = synth.make_workload("tiny")
    codes, scales = O.fp4_quantize(wl.kv_f32()[0])
    q = O.bf16_to_f64(wl.q(0)[0, 0])
    topk = np.array([777, -1, -1], np.int32)
    empty = np.zeros((0, q.shape[1]))
    out, _ = O.attention_unit(q, codes, scales, topk, empty, empty, 0, 2047, 0)
    g = O.fp4_dequantize(codes[777], scales[777])
    assert np.array_equal(out, np.broadcast_to(g, out.shape))


def test_union_and_overlap_fig4(golden):
    """With q = 0 every logit is equal, so out is the plain average of the union's values.
    Fig. 4's union has 4 entries; a position in both the global list and the window
    (the overlap case discussed under Fig. 4) is counted twice."""
    g4 = golden("fig4_selection.json")
    D = 16
    gvals = np.eye(6, D) * 12.0          # distinct, FP4-exact global rows p0..p5 (12 = 6 * 2)
    codes, scales = O.fp4_quantize(gvals.astype(np.float32))
    assert np.array_equal(O.fp4_dequantize(codes, scales), gvals)
    kl = np.zeros((6, D))
    vl = np.eye(6, D) * -1.0             # local values tell themselves apart from global ones
    q = np.zeros((1, D))
    out, lse = O.attention_unit(q, codes, scales, np.array(g4["expected_topk"]), kl, vl, 0, g4["t"], g4["W"])
    exp = (gvals[0] + gvals[3] + vl[4] + vl[5]) / g4["expected_entries"]
    assert np.array_equal(out[0], exp)
    assert abs(lse[0] - math.log(4)) < 1e-15
    out2, _ = O.attention_unit(q, codes, scales, np.array([0, 4]), kl, vl, 0, 5, 2)
    assert np.allclose(out2[0], (gvals[0] + gvals[4] + vl[4] + vl[5]) / 4, atol=0, rtol=0)


def test_window_bounds():
    assert O.window_positions(10, 4, 0).tolist() == [7, 8, 9, 10]
    assert O.window_positions(2, 4, 0).tolist() == [0, 1, 2]
    assert O.window_positions(10, 4, 9).tolist() == [9, 10]          # bounded replay truncation
    assert O.window_positions(10, 0, 0).tolist() == []
    assert O.window_positions(0, 1, 0).tolist() == [0]


def test_empty_union():
    out, lse = O.attend(np.ones((2, 8)), np.zeros((0, 8)), np.zeros((0, 8)), 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_bounded_replay_truncates_window_at_the_segment():
    """Bounded replay ("CED: Continuing Context with a Causal Encoder and Decoder",
    "Why Prefill Recomputes a Recent Segment", Fig. 6): only the last R prompt
    positions pass through the decoder again, and window references before the
    replayed segment are cut. With local_base = N - R the first replayed position
    reads only its own local row, and the last position (R = W) reads the same W
    rows as a full execution, so its output equals the untruncated one while the
    first position's does not."""
    wl = synth.make_workload("replay_prefill", B=1, N=3000, Tq=8, W=8, layers=synth.workloads._stack20_layers(64, 256)[:2])
    s = wl.spec
    assert s.local_base == s.N - s.Tq and s.Lloc == s.Tq
    assert O.window_positions(s.N - s.Tq, s.W, s.local_base).tolist() == [s.N - s.Tq]
    assert O.window_positions(s.N - 1, s.W, s.local_base).tolist() == list(range(s.N - s.W, s.N))
    codes, scales = O.fp4_quantize(wl.kv_f32()[0])
    rng = np.random.default_rng(3)
    q = rng.standard_normal((s.Hq, s.D))
    kl = rng.standard_normal((s.N, s.D))       # local rows of every position (a full execution's)
    vl = rng.standard_normal((s.N, s.D))
    topk = np.sort(rng.choice(s.N - s.Tq, 64, replace=False)).astype(np.int32)
    seg = slice(s.local_base, s.N)
    for t, same in ((s.N - 1, True), (s.N - s.Tq, False)):
        trunc = O.attention_unit(q, codes, scales, topk, kl[seg], vl[seg], s.local_base, t, s.W)
        full = O.attention_unit(q, codes, scales, topk, kl, vl, 0, t, s.W)
        assert np.allclose(trunc[0], full[0], rtol=0, atol=1e-12) == same
