"""Host logic of bench.py: the algorithmic byte count and the schedule label."""
import numpy as np

import bench
import synth


def _lists(spec, rng, dup=False):
    """Index lists of the right shapes for spec (ascending, -1 padded). With dup, the
    queries of a sequence share half of their entries."""
    B, Tq, N = spec.B, spec.Tq, spec.N
    pools, topks = [], []
    P_cur = 0
    for L in spec.layers:
        if L.mode == "REUSE":
            pools.append(None)
            topks.append(None)
            continue
        if L.mode == "FULL" and L.P:
            P_cur = L.P
        pool = np.full((B, Tq, max(P_cur, 1)), -1, np.int32) if (L.mode == "FULL" and L.P) else None
        topk = np.full((B, Tq, L.k), -1, np.int32)
        for b in range(B):
            shared = np.sort(rng.choice(N, L.k // 2, replace=False))
            for j in range(Tq):
                if dup:
                    rest = rng.choice(np.setdiff1d(np.arange(N), shared), L.k - L.k // 2, replace=False)
                    topk[b, j] = np.sort(np.concatenate([shared, rest]))
                else:
                    topk[b, j] = np.sort(rng.choice(N, L.k, replace=False))
                if pool is not None:
                    pool[b, j] = np.sort(rng.choice(N, L.P, replace=False))
        pools.append(pool)
        topks.append(topk)
    return pools, topks


def test_list_bytes_equal_per_query_sum_with_one_query_per_sequence():
    spec = synth.make_workload("stack20_128k").spec
    q_pos = np.full((spec.B, 1), spec.N - 1, np.int32)
    base = np.full((spec.B,), spec.N - spec.W, np.int32)
    pools, topks = _lists(spec, np.random.default_rng(1))
    assert bench.list_bytes(spec, q_pos, base, pools, topks) == bench.unit_bytes(spec) * spec.B
    assert bench.full_launch_bytes(spec, q_pos) == 134_881_280


def test_list_bytes_count_shared_rows_once():
    spec = synth.make_workload("tiny").spec            # 16 queries of one sequence
    q_pos = np.arange(spec.N - spec.Tq, spec.N, dtype=np.int32)[None, :]
    base = np.array([spec.N - spec.Tq - spec.W + 1], np.int32)
    rng = np.random.default_rng(2)
    pools, topks = _lists(spec, rng, dup=True)
    k = spec.layers[0].k
    got = bench.list_bytes(spec, q_pos, base, pools, topks)
    uniq = len(np.unique(topks[0][0]))
    assert uniq < spec.Tq * k                          # the lists overlap
    window_rows = (spec.N - 1) - (spec.N - spec.Tq - spec.W + 1) + 1   # union of the 16 windows
    want = (spec.N * spec.Di + spec.Tq * (spec.Hi * spec.Di + k * 4)          # Full call
            + uniq * (spec.D // 2 + spec.D // 16) + window_rows * 2 * spec.D * 2
            + spec.Tq * (k * 4 + 2 * spec.Hq * spec.D * 2))                    # attention call
    assert got == want


def test_window_union():
    assert bench._window_rows([0, 5, 20], [10, 12, 19]) == 13      # [0,12]; [20,19] is empty
    assert bench._window_rows([3, 14], [13, 20]) == 18              # adjacent intervals join
    assert bench._window_rows([], []) == 0


def test_schedule_labels():
    label = lambda w: bench.schedule_str(synth.make_workload(w).spec)
    assert label("stack20_128k") == "[F,U,U,RI]x5"
    assert label("paper_schedule") == "F,U,U,U," + "RI,U,U,U," * 3 + "RI,U,U,U"
    assert label("long_1m") == "F," + "RI,U," * 9 + "RI"
    assert label("decode_full") == "F"


def test_launch_count():
    count = lambda w: bench.launches_per_step(synth.make_workload(w).spec)
    assert count("stack20_128k") == 10 + 20          # 5 Full + 5 Reindex indexers, 20 attention launches
    assert count("long_1m") == 2 + 10 + 20           # the Full layer of 64 queries is scored first
    assert count("prefill_chunk") == 2 + 1
    assert count("tiny") == 1 + 1                    # 2048 keys: one indexer launch
