"""Plain CPU oracle for CSA2 sparse attention over a shared FP4 global KV cache.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import or run this module.
The GPU product path never calls it, and it shares no code with that path: it
has its own format tables, its own selection and its own softmax.

Sources (page titles; sections and figures named on each page):
  [CED]  "CED: Continuing Context with a Causal Encoder and Decoder"
         (ai-systems-engineering.com).
  [KVC]  "DeepSeek-V4.1 Flash Pushes KV Cache Compression for Agent Workloads"
         (news.puhulab.com), Turkish draft, section "Ana Gelişme".
  [OCP]  OCP Microscaling Formats (MX) Specification v1.0, the published
         definition of the E2M1 and E4M3 element formats that [KVC] names.

Arithmetic: scores are exact integers (int64), attention is fp64. All steps run
in the order the pages state them, one query at a time; a library sort or
matrix product serves as a single step where noted.

Parity status per function (what pins it is listed in the tests):
  e2m1_value, e4m3_value, fp4_quantize, fp4_dequantize   pinned
  index_scores, select_best, index_full, index_reindex    pinned
  window_positions, attend, attention_unit                pinned
  layer_stack_unit                                        pinned (invariants + Fig. 5)
  The score formula itself (sum over heads of w_h * relu(q_h . k)) is a reading
  of the pages, not something they state; its quality against a trained model
  is unpinned by construction.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

# --------------------------------------------------------------------------
# FP4 (E2M1) values with one E4M3 scale per 16 channels  [KVC]; formats [OCP]
# --------------------------------------------------------------------------


def e2m1_value(code) -> np.ndarray:
    """Value of a 4-bit E2M1 code: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.

    Exponent field 0 is subnormal: 0.5 * mantissa. No infinities or NaNs.
    """
    c = np.asarray(code, dtype=np.int64)
    sign = np.where((c >> 3) & 1, -1.0, 1.0)
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, (e - 1).astype(np.int32)))
    return sign * mag


def e4m3_value(byte) -> np.ndarray:
    """Value of an 8-bit E4M3 code: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.

    Exponent field 0 is subnormal: 2^-6 * m/8. Exponent 15 with mantissa 7 is NaN;
    no infinities. Largest finite value 448.
    """
    b = np.asarray(byte, dtype=np.int64)
    sign = np.where((b >> 7) & 1, -1.0, 1.0)
    e = (b >> 3) & 15
    m = b & 7
    sub = np.ldexp(m / 8.0, -6)
    nor = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int32))
    mag = np.where(e == 0, sub, nor)
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


# non-negative finite representable values, ascending, with their codes
_E2M1_POS_CODES = np.arange(8)
_E2M1_POS_VALUES = e2m1_value(_E2M1_POS_CODES)          # 0, .5, 1, 1.5, 2, 3, 4, 6
_E4M3_POS_CODES = np.arange(127)                        # 0x00 .. 0x7E
_E4M3_POS_VALUES = e4m3_value(_E4M3_POS_CODES)          # 0 .. 448


def _round_nearest_even(x: np.ndarray, values: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """Code of the representable value nearest to each x >= 0; a tie goes to the even code.

    Values above the largest representable value saturate to it.
    """
    x = np.asarray(x, dtype=np.float64)
    hi = np.searchsorted(values, x, side="left")          # first value >= x
    hi = np.clip(hi, 0, len(values) - 1)
    lo = np.clip(hi - 1, 0, len(values) - 1)
    d_lo = np.abs(x - values[lo])
    d_hi = np.abs(values[hi] - x)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (codes[hi] % 2 == 0))
    out = np.where(pick_hi, codes[hi], codes[lo])
    return np.where(x >= values[-1], codes[-1], out)


def e4m3_round(x) -> np.ndarray:
    """E4M3 code nearest to x >= 0 (ties to even), saturating at 448."""
    return _round_nearest_even(x, _E4M3_POS_VALUES, _E4M3_POS_CODES).astype(np.uint8)


def e2m1_round(x) -> np.ndarray:
    """E2M1 code nearest to x (ties to even), saturating at +-6; never emits -0."""
    x = np.asarray(x, dtype=np.float64)
    mag_code = _round_nearest_even(np.abs(x), _E2M1_POS_VALUES, _E2M1_POS_CODES)
    neg = (x < 0) & (mag_code != 0)
    return (mag_code + 8 * neg).astype(np.uint8)


def fp4_quantize(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Quantise rows of fp32 values to FP4 with one E4M3 scale per 16 channels.

    x: [..., D] float32, D % 16 == 0.
    Returns codes uint8 [..., D/2] (element 2j in the low nibble, 2j+1 in the high
    nibble) and scales uint8 [..., D/16] (E4M3 bit patterns).

    Per group of 16: amax = max |x|; the scale is the E4M3 value nearest amax/6
    (so the largest element maps to the largest E2M1 magnitude, 6), ties to even,
    saturating at 448; each code is the E2M1 value nearest x/scale, ties to even,
    saturating at +-6. A zero scale (amax/6 rounds to 0) gives all-zero codes.
    Both roundings are decided on the exact quotient: fp64 division of an fp32 by a
    value with at most 4 significant bits cannot move a quotient across a rounding
    boundary of these formats, so fp64 gives the same decisions.
    """
    x = np.asarray(x, dtype=np.float32)
    D = x.shape[-1]
    assert D % 16 == 0
    g = x.reshape(-1, D // 16, 16).astype(np.float64)
    amax = np.abs(g).max(axis=-1)
    s_code = e4m3_round(amax / 6.0)
    s = e4m3_value(s_code)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(s[..., None] > 0, g / np.where(s > 0, s, 1.0)[..., None], 0.0)
    codes = e2m1_round(r).reshape(-1, D)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed.reshape(x.shape[:-1] + (D // 2,)), s_code.reshape(x.shape[:-1] + (D // 16,))


def fp4_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """fp64 values of FP4 rows: e2m1(code) * e4m3(scale of the element's 16-group)."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    D = codes.shape[-1] * 2
    lo = codes & 0x0F
    hi = codes >> 4
    elem = np.empty(codes.shape[:-1] + (D,), dtype=np.int64)
    elem[..., 0::2] = lo
    elem[..., 1::2] = hi
    scale = np.repeat(e4m3_value(scales), 16, axis=-1)
    return e2m1_value(elem) * scale


# --------------------------------------------------------------------------
# Indexer: Full / Reindex / Reuse   [CED] "Selecting Positions and Reading
# Values with Attention" (Fig. 4) and "What Full, Reindex, and Reuse Share" (Fig. 5)
# --------------------------------------------------------------------------


def index_scores(qi: np.ndarray, w: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """score(s) = sum_h w[h] * max(0, sum_d qi[h, d] * keys[s, d]), exact int64.

    qi [Hi, Di] int8, w [Hi] int, keys [n, Di] int8 -> [n] int64.
    The dot products are one fp64 matrix product: every partial sum is an integer
    of magnitude below Di * 128 * 128 < 2^53, so the product is exact.
    """
    qi = np.asarray(qi, dtype=np.int64)
    keys = np.asarray(keys, dtype=np.int64)
    assert qi.shape[1] * 128 * 128 < 2 ** 53
    dots = (keys.astype(np.float64) @ qi.astype(np.float64).T).astype(np.int64)   # [n, Hi]
    relu = np.maximum(dots, 0)
    return relu @ np.asarray(w, dtype=np.int64)


def select_best(scores: np.ndarray, positions: np.ndarray, count: int) -> np.ndarray:
    """The `count` candidates ranked first by (score descending, position ascending),
    returned in ascending position order."""
    scores = np.asarray(scores, dtype=np.int64)
    positions = np.asarray(positions, dtype=np.int64)
    order = np.lexsort((positions, -scores))
    return np.sort(positions[order[:count]])


def pad_list(pos: np.ndarray, length: int) -> np.ndarray:
    out = np.full((length,), -1, dtype=np.int32)
    out[: len(pos)] = pos
    return out


def last_entry(t: int, m: int = 1) -> int:
    """The last global entry the query at position t may read. With sequence
    compression rate m >= 2, entry j combines positions m*j .. m*j + m - 1 ([CED]
    "What Does the Sequence Compression Rate Reduce?": two positions become one
    entry at m = 2; the teaching example counts only complete groups), so it is
    readable once position m*j + m - 1 <= t. With m = 1 entries are positions."""
    if m <= 1:
        return t
    return (t + 1) // m - 1


def valid_positions(t: int, N: int, m: int = 1) -> np.ndarray:
    """Causal candidates of the query at position t: entries 0 <= s <= last_entry(t)
    and s < N ([CED] "One Token Sequence and Causal Access", Fig. 2)."""
    return np.arange(0, min(last_entry(t, m), N - 1) + 1, dtype=np.int64)


def compress_entries(x: np.ndarray, m: int) -> np.ndarray:
    """Global entries of compression rate m from per-position rows x [n, D] (n a
    multiple of m): entry g combines rows g*m .. g*m + m - 1. The pages give no
    combining rule (PARITY UNPINNED for the rule itself); this reading takes the
    mean, summed left to right in fp32 and scaled by 1/m, which is exact for m a
    power of two."""
    x = np.asarray(x, dtype=np.float32)
    g = x.reshape(x.shape[:-2] + (x.shape[-2] // m, m, x.shape[-1]))
    acc = g[..., 0, :].copy()
    for r in range(1, m):
        acc = (acc + g[..., r, :]).astype(np.float32)
    return (acc * np.float32(1.0 / m)).astype(np.float32)


def index_full(qi, w, keys_seq, t: int, k: int, P: int = 0, m: int = 1):
    """Full mode: score every causal position, keep the top-P pool and the top-k list.

    keys_seq [N, Di] int8 of the query's sequence. Returns (pool or None, topk),
    each padded with -1 to its length. topk is the top-k of the same scores, so it
    is a subset of the pool ([CED] Fig. 5, "Hierarchical Sparse Indexer").
    """
    cand = valid_positions(t, keys_seq.shape[0], m)
    sc = index_scores(qi, w, keys_seq[cand])
    topk = pad_list(select_best(sc, cand, k), k)
    pool = pad_list(select_best(sc, cand, P), P) if P > 0 else None
    return pool, topk


def index_reindex(qi, w, keys_seq, pool_in: np.ndarray, k: int) -> np.ndarray:
    """Reindex mode: rescore only the candidate pool with this layer's own indexer
    query and keys, and keep its top-k ([CED] Fig. 5)."""
    cand = np.asarray(pool_in, dtype=np.int64)
    cand = cand[cand >= 0]
    sc = index_scores(qi, w, keys_seq[cand])
    return pad_list(select_best(sc, cand, k), k)


# --------------------------------------------------------------------------
# Core attention over {selected global rows} U {local window}
# [CED] "Selecting Positions and Reading Values with Attention" (Fig. 4)
# --------------------------------------------------------------------------


def window_positions(t: int, W: int, local_base: int) -> np.ndarray:
    """Positions of the query's sliding window: [max(local_base, t-W+1, 0), t];
    empty when W == 0. The current position is included (causal access allows it)."""
    if W <= 0:
        return np.zeros((0,), dtype=np.int64)
    lo = max(local_base, t - W + 1, 0)
    return np.arange(lo, t + 1, dtype=np.int64)


def attend(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float):
    """One softmax over all given entries, per head, in fp64.

    q [Hq, D], keys/values [n, D]. Returns out [Hq, D], lse [Hq] (natural log of
    the sum of exp(logits)). With no entries, out is 0 and lse is -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    if keys.shape[0] == 0:
        return np.zeros_like(q), np.full((q.shape[0],), -np.inf)
    logits = (q @ np.asarray(keys, np.float64).T) * scale            # [Hq, n]
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    out = (p @ np.asarray(values, np.float64)) / l
    return out, (m + np.log(l))[:, 0]


def attention_unit(q, kv_codes_seq, kv_scales_seq, topk, kl_seq, vl_seq,
                   local_base: int, t: int, W: int, scale: Optional[float] = None):
    """Attention of one query (all heads) over its selected global rows and window.

    Global rows are dequantised FP4 and serve as both key and value (one vector per
    position). Local rows use their own K and V. A position in both sets is counted
    twice: the two entries come from different paths ([CED] Fig. 4 discussion).
    q [Hq, D] (fp64 values of the bf16 inputs); kv_*_seq: the sequence's cache;
    topk: the layer's list (-1 padded); kl_seq/vl_seq [Lloc, D] fp64.
    """
    D = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    sel = np.asarray(topk, dtype=np.int64)
    sel = sel[sel >= 0]
    g = fp4_dequantize(kv_codes_seq[sel], kv_scales_seq[sel])
    win = window_positions(t, W, local_base) - local_base
    keys = np.concatenate([g, kl_seq[win]], axis=0)
    vals = np.concatenate([g, vl_seq[win]], axis=0)
    return attend(q, keys, vals, scale)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """fp64 value of bf16 bit patterns (the top 16 bits of an fp32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)



# --------------------------------------------------------------------------
# Layer stack over one shared cache   [CED] "What Full, Reindex, and Reuse Share"
# --------------------------------------------------------------------------

FULL, REINDEX, REUSE = "FULL", "REINDEX", "REUSE"


def layer_stack_unit(layers: Sequence[dict], t: int, kv_codes_seq, kv_scales_seq,
                     local_base: int, with_attention: bool = True, m: int = 1) -> List[Dict]:
    """Run the decoder layers for one query at position t.

    Each entry of `layers` is a dict with
      mode: FULL | REINDEX | REUSE
      FULL:    qi [Hi,Di], w [Hi], keys [N,Di], k, P
      REINDEX: qi, w, keys, k          (rescores the most recent Full layer's pool)
      all:     q [Hq,D] fp64, kl [Lloc,D] fp64, vl [Lloc,D] fp64, W
    Reuse takes the list of the most recent Full or Reindex layer unchanged; every
    layer still attends with its own main query and local KV.
    Returns per layer {mode, pool, topk, out, lse}.
    """
    res: List[Dict] = []
    pool = None
    cur = None
    for li, L in enumerate(layers):
        mode = L["mode"]
        entry = {"mode": mode, "pool": None}
        if mode == FULL:
            pool_l, cur = index_full(L["qi"], L["w"], L["keys"], t, L["k"], L.get("P", 0), m)
            if pool_l is not None:
                pool = pool_l
            entry["pool"] = pool_l
        elif mode == REINDEX:
            if pool is None:
                raise ValueError(f"layer {li}: REINDEX needs a pool from an earlier FULL layer")
            cur = index_reindex(L["qi"], L["w"], L["keys"], pool, L["k"])
        elif mode == REUSE:
            if cur is None:
                raise ValueError(f"layer {li}: REUSE needs an earlier FULL or REINDEX layer")
            cur = cur.copy()
        else:
            raise ValueError(mode)
        entry["topk"] = cur
        if with_attention:
            entry["out"], entry["lse"] = attention_unit(
                L["q"], kv_codes_seq, kv_scales_seq, cur, L["kl"], L["vl"], local_base, t, L["W"])
        res.append(entry)
    return res
