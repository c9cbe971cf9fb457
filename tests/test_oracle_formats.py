"""Pins of the oracle's FP4 (E2M1) / E4M3 arithmetic against things other than itself:
a library cast (torch float8_e4m3fn), the published E2M1 table, brute-force nearest
search, and exact round trips on grid values."""
import itertools

import numpy as np
import pytest
import torch

import synth
from oracle import csa2_oracle as O


def test_e4m3_table_matches_torch_cast():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = O.e4m3_value(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(mine))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], mine[ok])
    assert np.array_equal(np.signbit(ref[ok]), np.signbit(mine[ok]))


def test_e2m1_table_matches_published_values(golden):
    g = golden("e2m1_values.json")
    mine = O.e2m1_value(np.array(g["codes"]))
    assert np.array_equal(mine, np.array(g["values"]))
    assert np.array_equal(np.signbit(mine), np.signbit(np.array(g["values"])))


def _e4m3_pos_values():
    v = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return v


def test_e4m3_round_matches_torch_cast_in_range():
    vals = _e4m3_pos_values()
    mids = (vals[:-1] + vals[1:]) / 2                       # every tie
    rng = np.random.default_rng(0)
    rand = np.concatenate([rng.uniform(0, 448, 20000), np.exp(rng.uniform(np.log(1e-4), np.log(448), 20000))])
    near = np.concatenate([mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20)])
    x = np.concatenate([vals, mids, rand, near, [0.0, 2.0 ** -10, 1e-9]]).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_round(x), ref)


def test_e4m3_round_saturates():
    assert np.all(O.e4m3_round(np.array([448.0, 449.0, 470.0, 1e6])) == 0x7E)


def _brute_e2m1(x):
    """Nearest E2M1 code by exhaustive search over all 16 codes; ties to the even code;
    -0 never returned."""
    best = None
    for c in range(16):
        if c == 8:
            continue
        v = float(O.e2m1_value(c))
        d = abs(x - v)
        key = (d, (c & 7) % 2, c)           # smaller error, then even magnitude code
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_e2m1_round_bruteforce():
    grid = [float(v) for v in O.e2m1_value(np.arange(8))]
    pts = set()
    for a, b in zip(grid[:-1], grid[1:]):
        m = (a + b) / 2
        pts.update([a, b, m, m + 1e-6, m - 1e-6])
    pts.update([6.5, 7.0, 100.0, 1e-9])
    rng = np.random.default_rng(1)
    pts.update(rng.uniform(-7, 7, 3000).tolist())
    xs = np.array(sorted(pts | {-p for p in pts}))
    got = O.e2m1_round(xs)
    exp = np.array([_brute_e2m1(x) for x in xs])
    # saturation: beyond 6 the brute force also picks 6 (nearest)
    assert np.array_equal(got, exp)


def test_e2m1_ties_golden(golden):
    g = golden("e2m1_rne_ties.json")
    got = O.e2m1_value(O.e2m1_round(np.array(g["inputs"])))
    assert np.array_equal(got, np.array(g["expected"]))


def test_quantize_scale_is_nearest_e4m3_of_amax_over_6():
    x = synth.normal_f32(0, 11, (64, 128))
    _, s = O.fp4_quantize(x)
    vals = _e4m3_pos_values()
    amax = np.abs(x.reshape(64, 8, 16).astype(np.float64)).max(-1)
    for (r, g), code in np.ndenumerate(s):
        target = amax[r, g] / 6
        d = np.abs(vals - target)
        best = np.flatnonzero(d == d.min())
        best = best[best % 2 == 0] if len(best) > 1 else best
        assert code == best[0]


def test_quantize_codes_are_nearest_bruteforce():
    x = synth.normal_f32(0, 12, (16, 64))
    codes, scales = O.fp4_quantize(x)
    s = O.e4m3_value(scales)                                # [16, 4]
    for r in range(16):
        for d in range(64):
            c = (codes[r, d // 2] >> (4 * (d % 2))) & 15
            assert c == _brute_e2m1(float(x[r, d]) / s[r, d // 16]), (r, d)


def test_roundtrip_exact_on_grid_blocks():
    """Blocks whose values are e2m1 * s with s an E4M3 value and one element at +-6s
    quantise back to themselves exactly (amax/6 = s exactly)."""
    rng = np.random.default_rng(2)
    e4 = _e4m3_pos_values()[1:]                      # non-zero scales
    e4 = e4[e4 * 6 < 3.0e38]
    rows = []
    for i in range(500):
        s = e4[rng.integers(0, len(e4))]
        codes = rng.integers(0, 16, 16)
        codes[codes == 8] = 0
        codes[rng.integers(0, 16)] = 7 if rng.random() < 0.5 else 15
        rows.append(O.e2m1_value(codes) * s)
    x = np.array(rows, dtype=np.float64).reshape(-1, 32)
    assert np.array_equal(x.astype(np.float32).astype(np.float64), x)
    c, sc = O.fp4_quantize(x.astype(np.float32))
    assert np.array_equal(O.fp4_dequantize(c, sc), x)


def test_dequantized_values_are_exact_in_bf16():
    e2 = O.e2m1_value(np.arange(16))
    e4 = O.e4m3_value(np.arange(256))
    prod = np.outer(e2, e4[~np.isnan(e4)]).ravel()
    as_bf16 = torch.from_numpy(prod).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(as_bf16, prod)


def test_zero_group_gives_zero_scale_and_codes():
    x = np.zeros((2, 32), dtype=np.float32)
    x[1, 16:] = 1e-4                                   # amax/6 below half the smallest subnormal
    c, s = O.fp4_quantize(x)
    assert np.all(s == 0) and np.all(c == 0)
    assert np.all(O.fp4_dequantize(c, s) == 0)


def test_fp4_bytes_per_token():
    """Global KV bytes per position: D/2 code bytes + D/16 scale bytes (72 at D=128)."""
    x = synth.normal_f32(0, 13, (3, 128))
    c, s = O.fp4_quantize(x)
    assert c.shape[-1] + s.shape[-1] == 72


def test_bf16_to_f64_every_pattern():
    """The oracle's bf16 decoding against torch's bfloat16 -> float64 conversion, for all
    65536 bit patterns (NaN patterns decode to NaN on both sides)."""
    import torch
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):      # signalling-NaN patterns
        ours = O.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))   # -0 stays -0
