"""Pins of the oracle's indexer (scores, exact top-k, Full/Reindex) against brute force in
plain Python integers, adversarial ties, the pages' worked examples (Fig. 4, Fig. 5) and
the invariants the pages state (causality, Reindex within the pool)."""
import itertools

import numpy as np
import pytest

import synth
from oracle import csa2_oracle as O


def _py_scores(qi, w, keys):
    out = []
    for row in keys.tolist():
        tot = 0
        for h, qh in enumerate(qi.tolist()):
            dot = sum(a * b for a, b in zip(qh, row))
            tot += int(w[h]) * max(0, dot)
        out.append(tot)
    return out


def _py_select(scores, positions, count):
    ranked = sorted(zip(scores, positions), key=lambda sp: (-sp[0], sp[1]))
    return sorted(p for _, p in ranked[:count])


@pytest.mark.parametrize("seed", range(6))
def test_scores_match_python_integers(seed):
    rng = np.random.default_rng(seed)
    Hi, Di, n = rng.integers(1, 9), int(rng.integers(1, 5) * 8), 40
    qi = rng.integers(-128, 128, (Hi, Di)).astype(np.int8)       # -128 included on purpose
    keys = rng.integers(-128, 128, (n, Di)).astype(np.int8)
    w = rng.integers(-8, 9, Hi)
    assert O.index_scores(qi, w, keys).tolist() == _py_scores(qi, w, keys)


def test_scores_extreme_magnitudes():
    qi = np.full((8, 64), -128, np.int8)
    keys = np.full((3, 64), -128, np.int8)
    w = np.full(8, 255)
    assert O.index_scores(qi, w, keys).tolist() == [8 * 255 * 64 * 128 * 128] * 3


@pytest.mark.parametrize("seed", range(4))
def test_select_bruteforce_all_k(seed):
    rng = np.random.default_rng(100 + seed)
    n = 30
    scores = rng.integers(0, 6, n)                  # many ties
    pos = np.sort(rng.choice(1000, n, replace=False))
    for k in range(0, n + 3):
        assert O.select_best(scores, pos, k).tolist() == _py_select(scores.tolist(), pos.tolist(), k)


@pytest.mark.parametrize("seed", range(3))
def test_full_bruteforce_tiny(seed):
    rng = np.random.default_rng(200 + seed)
    N, Hi, Di = 48, 3, 16
    keys = rng.integers(-127, 128, (N, Di)).astype(np.int8)
    qi = rng.integers(-127, 128, (Hi, Di)).astype(np.int8)
    w = rng.integers(1, 9, Hi)
    for t in [0, 1, 5, 30, 47]:
        for k in [1, 2, 7, 64]:
            for P in [0, k, k + 5]:
                pool, topk = O.index_full(qi, w, keys, t, k, P)
                cand = list(range(t + 1))
                sc = _py_scores(qi, w, keys[: t + 1])
                exp = _py_select(sc, cand, k)
                assert topk.tolist() == exp + [-1] * (k - len(exp))
                if P:
                    expp = _py_select(sc, cand, P)
                    assert pool.tolist() == expp + [-1] * (P - len(expp))
                    assert set(exp) <= set(expp)


def test_all_equal_scores_pick_lowest_positions():
    keys = np.full((100, 32), 3, np.int8)
    qi = synth.randint_i8(0, 1, (4, 32))
    w = np.array([1, 2, 3, 4])
    _, topk = O.index_full(qi, w, keys, 99, 10, 0)
    assert topk.tolist() == list(range(10))


def test_relu_zero_scores_pick_lowest_positions():
    keys = np.full((50, 16), -127, np.int8)
    qi = np.full((2, 16), 100, np.int8)
    pool, topk = O.index_full(qi, np.array([5, 7]), keys, 40, 4, 8)
    assert topk.tolist() == [0, 1, 2, 3]
    assert pool.tolist() == list(range(8))


def test_causal_triangle_and_counts():
    wl = synth.make_workload("tiny")
    keys = wl.ki(0)[0]
    for t in [0, 3, 255, 256, 1000, 2047]:
        pool, topk = O.index_full(wl.qi(0)[0, 0], wl.w(0), keys, t, 256, 512)
        valid = topk[topk >= 0]
        assert len(valid) == min(256, t + 1)
        assert np.all(valid <= t) and np.all(np.diff(valid) > 0)
        assert np.all(topk[len(valid):] == -1)
        assert set(valid.tolist()) <= set(pool[pool >= 0].tolist())


def test_fig4_selection(golden):
    g = golden("fig4_selection.json")
    keys = np.array(g["keys"], np.int8)
    _, topk = O.index_full(np.array(g["qi"], np.int8), np.array(g["w"]), keys, g["t"], g["k"], 0)
    assert topk.tolist() == g["expected_topk"]
    assert O.window_positions(g["t"], g["W"], g["local_base"]).tolist() == g["expected_window"]


def test_fig5_full_reindex_reuse(golden):
    g = golden("fig5_modes.json")
    f, r = g["full"], g["reindex"]
    pool, topk = O.index_full(np.array(f["qi"], np.int8), np.array(f["w"]), np.array(f["keys"], np.int8),
                              g["t"], g["k"], g["P"])
    assert pool.tolist() == g["expected_full_pool"]
    assert topk.tolist() == g["expected_full_topk"]
    ri = O.index_reindex(np.array(r["qi"], np.int8), np.array(r["w"]), np.array(r["keys"], np.int8), pool, g["k"])
    assert ri.tolist() == g["expected_reindex_topk"]
    # stack form: Full -> Reindex -> Reuse
    layers = [
        {"mode": "FULL", "qi": np.array(f["qi"], np.int8), "w": np.array(f["w"]), "keys": np.array(f["keys"], np.int8),
         "k": g["k"], "P": g["P"]},
        {"mode": "REINDEX", "qi": np.array(r["qi"], np.int8), "w": np.array(r["w"]), "keys": np.array(r["keys"], np.int8),
         "k": g["k"]},
        {"mode": "REUSE"},
    ]
    res = O.layer_stack_unit(layers, g["t"], None, None, 0, with_attention=False)
    assert [e["topk"].tolist() for e in res] == [g["expected_full_topk"], g["expected_reindex_topk"],
                                                 g["expected_reuse_topk"]]


def test_reindex_with_full_pool_and_same_inputs_equals_full():
    wl = synth.make_workload("tiny")
    keys, qi, w = wl.ki(0)[0], wl.qi(0)[0, 3], wl.w(0)
    t = 1500
    pool, topk = O.index_full(qi, w, keys, t, 200, 2048)       # pool = every causal position
    assert (pool >= 0).sum() == t + 1
    assert np.array_equal(O.index_reindex(qi, w, keys, pool, 200), topk)


def test_reindex_subset_of_pool():
    wl = synth.make_workload("tiny")
    pool, _ = O.index_full(wl.qi(0)[0, 0], wl.w(0), wl.ki(0)[0], 2047, 64, 300)
    other_keys = synth.randint_i8(0, 999, (2048, 32))
    ri = O.index_reindex(synth.randint_i8(0, 998, (4, 32)), np.array([1, 1, 1, 1]), other_keys, pool, 64)
    assert set(ri.tolist()) <= set(pool.tolist())
    assert len(set(ri.tolist()) - set(O.index_full(wl.qi(0)[0, 0], wl.w(0), wl.ki(0)[0], 2047, 64)[1].tolist())) > 0


def test_stack_errors():
    with pytest.raises(ValueError):
        O.layer_stack_unit([{"mode": "REUSE"}], 3, None, None, 0, with_attention=False)
    keys = np.zeros((4, 8), np.int8)
    with pytest.raises(ValueError):
        O.layer_stack_unit([{"mode": "FULL", "qi": np.zeros((1, 8), np.int8), "w": [1], "keys": keys, "k": 2, "P": 0},
                            {"mode": "REINDEX", "qi": np.zeros((1, 8), np.int8), "w": [1], "keys": keys, "k": 2}],
                           3, None, None, 0, with_attention=False)


def test_paper_schedule_counts():
    spec = synth.CONFIGS["paper_schedule"]
    modes = [l.mode for l in spec.layers]
    assert (modes.count("FULL"), modes.count("REINDEX"), modes.count("REUSE")) == (1, 4, 15)
    assert modes[:4] == ["FULL", "REUSE", "REUSE", "REUSE"] and len(modes) == 20
