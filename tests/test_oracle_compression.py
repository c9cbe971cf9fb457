"""Pins of the oracle's sequence compression rate m ("CED: Continuing Context with a
Causal Encoder and Decoder", "What Does the Sequence Compression Rate Reduce?"):
the entry count of the page's worked example, the causal rule for a group of m
positions (brute force over positions), and the combining rule's reading (the
mean), which reduces to the identity at m = 1 and to the row itself for equal
rows. The combining rule itself is not on the pages: parity unpinned."""
import numpy as np
import pytest

import synth
from oracle import cpp as C
from oracle import csa2_oracle as O


def test_entry_counts_of_the_worked_example(golden):
    for case in golden("compression_rate.json")["cases"]:
        x = np.zeros((case["positions"], 16), np.float32)
        assert O.compress_entries(x, case["m"]).shape[0] == case["entries"]
        assert C.compress_entries(x, case["m"]).shape[0] == case["entries"]


@pytest.mark.parametrize("m", [1, 2, 4])
def test_last_entry_is_the_last_complete_group(m):
    for t in range(0, 40):
        readable = [j for j in range(40) if all(p <= t for p in range(m * j, m * j + m))]
        last = readable[-1] if readable else -1
        assert O.last_entry(t, m) == last
        assert C.lib().orc_last_entry(t, m) == last


def test_compress_is_identity_at_m1_and_keeps_equal_pairs():
    x = synth.normal_f32(4, 1, (64, 32))
    assert np.array_equal(O.compress_entries(x, 1), x)
    pairs = np.repeat(x, 2, axis=0)                       # positions 2j and 2j+1 hold the same row
    assert np.array_equal(O.compress_entries(pairs, 2), x)
    assert np.array_equal(C.compress_entries(pairs, 2), x)


def test_compress_mean_matches_exact_arithmetic_and_the_cpp_oracle():
    x = synth.normal_f32(4, 2, (2, 256, 128))
    for m in (2, 4):
        e = O.compress_entries(x, m)
        exact = x.astype(np.float64).reshape(2, 256 // m, m, 128).mean(axis=2)
        assert np.abs(e - exact).max() < 1e-6 * (1 + np.abs(exact).max())
        assert np.array_equal(C.compress_entries(x, m), e)


def test_full_over_entries_bruteforce():
    rng = np.random.default_rng(5)
    keys = rng.integers(-127, 128, (30, 16)).astype(np.int8)
    qi = rng.integers(-127, 128, (2, 16)).astype(np.int8)
    w = np.array([3, 1])
    sc = O.index_scores(qi, w, keys)
    for t in range(0, 60, 7):
        last = (t + 1) // 2 - 1
        cand = [j for j in range(30) if j <= last]
        ref = sorted(sorted(cand, key=lambda j: (-sc[j], j))[:5])
        _, topk = O.index_full(qi, w, keys, t, 5, 0, m=2)
        assert topk[topk >= 0].tolist() == ref
        _, t2 = C.index_full(qi, w, keys, O.last_entry(t, 2), 5)
        assert np.array_equal(t2, topk)
