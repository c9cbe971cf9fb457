"""The shared input generator: determinism, ranges, slice consistency, distribution."""
import numpy as np

import synth


def test_deterministic_and_slices_agree():
    a = synth.randint_i8(0, 5, (1000,))
    b = synth.randint_i8(0, 5, (1000,))
    assert np.array_equal(a, b)
    part = synth.randint_i8(0, 5, (300,), start=500)
    assert np.array_equal(a[500:800], part)
    n1 = synth.normal_f32(3, 9, (4000,))
    assert np.array_equal(n1[1000:2000], synth.normal_f32(3, 9, (1000,), start=1000))


def test_streams_differ():
    assert not np.array_equal(synth.randint_i8(0, 1, (64,)), synth.randint_i8(0, 2, (64,)))
    assert not np.array_equal(synth.randint_i8(0, 1, (64,)), synth.randint_i8(1, 1, (64,)))


def test_ranges():
    x = synth.randint_i8(0, 7, (200000,), -127, 127)
    assert x.min() == -127 and x.max() == 127
    w = synth.randint_i32(0, 8, (10000,), 1, 8)
    assert w.min() == 1 and w.max() == 8


def test_normal_moments_and_bf16():
    x = synth.normal_f32(0, 3, (400000,)).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    b = synth.normal_bf16(0, 3, (1000,))
    f = synth.normal_f32(0, 3, (1000,))
    back = (b.astype(np.uint32) << 16).view(np.float32)
    assert np.all(np.abs(back - f) <= np.abs(f) * 2.0 ** -8 + 1e-30)


def test_workload_shapes():
    wl = synth.make_workload("tiny")
    s = wl.spec
    assert (s.local_base, s.Lloc) == (1905, 143)
    assert wl.q_pos()[0].tolist() == list(range(2032, 2048))
    assert wl.q(0).shape == (1, 16, 8, 64) and wl.kl(0).shape == (1, 143, 64)
    st = synth.CONFIGS["stack20_128k"]
    modes = [l.mode for l in st.layers]
    assert modes[:4] == ["FULL", "REUSE", "REUSE", "REINDEX"] and len(modes) == 20
    assert st.n_key_sets == 10 and st.Lloc == 512
    lm = synth.CONFIGS["long_1m"]
    assert [l.mode for l in lm.layers[:4]] == ["FULL", "REINDEX", "REUSE", "REINDEX"]
    assert sum(l.mode == "REINDEX" for l in lm.layers) == 10 and lm.n_key_sets == 1
    pc = synth.CONFIGS["prefill_chunk"]
    assert (pc.local_base, pc.Lloc) == (65025, 4607)
