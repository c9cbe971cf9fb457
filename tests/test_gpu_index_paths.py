"""Every dispatch path of the indexer that the boundary accepts, against the oracle.

csa2_index_topk picks a kernel by mode, key width Di, head count Hi and the number
of queries per sequence: the tensor-core Full scan for Di in {32, 64, 128}
(preceded by the multi-query scoring kernel when Tq >= 4 queries share N >= 8192
keys with Hi <= 8), and dp4a kernels for Reindex and for Full with other key widths
(specialised for Hi <= 8 with Di = 64 and Hi <= 4 with Di = 32, generic otherwise).
Each case here runs one of them with inputs that include the int8 extreme -128
and head weights at the header's bound (Hi * max|w| * Di * 16384 < 2^31), and
checks every list bit-exactly against the oracle and for the causal layout
([CED] "One Token Sequence and Causal Access", Fig. 2; "What Full, Reindex, and
Reuse Share", Fig. 5)."""
import numpy as np
import pytest

import synth
from oracle import csa2_oracle as O
from sparse_attention_shared_b200 import ops

from gpu_util import assert_list_invariants, assert_lists_equal, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ws():
    return ops.Workspace()


@pytest.fixture
def status():
    s = ops.Status()
    yield s
    s.check("after test")


def max_weight(Hi, Di):
    """Largest |w| the header accepts for these sizes."""
    return ((1 << 31) - 1) // (Hi * Di * 16384)


def inputs(seed, B, Tq, N, Hi, Di, extreme):
    lo = -128 if extreme else -127
    qi = synth.randint_i8(seed, 1, (B, Tq, Hi, Di), lo, 127)
    ki = synth.randint_i8(seed, 2, (B, N, Di), lo, 127)
    if extreme:
        wm = max_weight(Hi, Di)
        w = synth.randint_i32(seed, 3, (Hi,), -wm, wm)
        w[0], w[-1] = wm, -wm
        qi[:, :, 0, :] = -128          # one head entirely at the extreme
        ki[:, ::97, :] = -128          # and some keys: dot products of 128 * 128 * Di
    else:
        w = synth.randint_i32(seed, 3, (Hi,), 1, 8)
    return qi, w, ki


def full_ref(qi, w, ki, q_pos, k, P):
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


def check_full(qi, w, ki, q_pos, k, P, ws, status):
    pool, topk = ops.index_topk("FULL", dev(q_pos), dev(qi), w, dev(ki), k, P, ws=ws, status=status)
    status.check("full")
    rpool, rtopk = full_ref(qi, w, ki, q_pos, k, P)
    assert_list_invariants(topk.cpu().numpy(), q_pos, "topk")
    assert_lists_equal(topk, rtopk, "topk")
    if P:
        assert_list_invariants(pool.cpu().numpy(), q_pos, "pool")
        assert_lists_equal(pool, rpool, "pool")
    return pool, topk


# (B, Tq, N, Hi, Di, k, P, extreme): the kernel each case reaches is in the comment
FULL_CASES = [
    (2, 1, 20000, 8, 128, 512, 2048, False),    # tensor-core scan, Di = 128, one query per sequence
    (2, 2, 9000, 8, 128, 300, 1000, True),      # ... two queries, -128 and extreme weights
    (1, 3, 12000, 6, 128, 256, 0, False),       # ... three queries, just under the multi-query cut-over
    (3, 3, 8192, 8, 64, 256, 1024, True),       # Di = 64, Tq = 3 on 8192 keys (not the multi-query path)
    (2, 1, 30000, 12, 64, 1024, 4096, False),   # 12 heads: the second TMEM column group of the scan
    (2, 2, 9000, 16, 64, 300, 1000, True),      # 16 heads, extremes
    (2, 1, 7000, 16, 32, 200, 800, True),       # Di = 32, 16 heads
    (2, 1, 10000, 8, 48, 512, 2048, False),     # Di = 48: generic-width dp4a Full path
    (2, 2, 6000, 5, 96, 300, 900, True),        # Di = 96: generic dp4a, extremes
    (1, 1, 3000, 16, 112, 100, 0, True),        # Di = 112, 16 heads, no pool
    (1, 1, 3000, 3, 16, 64, 128, True),         # Di = 16, the smallest width
    (2, 6, 9000, 8, 64, 300, 1000, True),       # multi-query scoring (Tq >= 4, N >= 8192) with extremes
    (1, 5, 8192, 4, 32, 128, 512, True),        # multi-query scoring, Di = 32
]


@pytest.mark.parametrize("B,Tq,N,Hi,Di,k,P,extreme", FULL_CASES)
def test_full_paths(B, Tq, N, Hi, Di, k, P, extreme, ws, status):
    qi, w, ki = inputs(B * 131 + N + Di, B, Tq, N, Hi, Di, extreme)
    rng = np.random.default_rng(N + Tq)
    q_pos = np.sort(rng.integers(N // 2, N, size=(B, Tq)), axis=1).astype(np.int32)
    q_pos[:, -1] = N - 1
    check_full(qi, w, ki, q_pos, k, P, ws, status)


# (B, N, Hi, Di, P, k, extreme): Reindex kernels (dp4a): <8,64>, <4,32>, generic
REINDEX_CASES = [
    (3, 12000, 8, 64, 4096, 1024, True),        # <8,64>, one select per group, extremes
    (2, 9000, 4, 32, 2048, 300, True),          # <4,32>
    (2, 9000, 12, 64, 2048, 500, True),         # generic (Hi > 8)
    (2, 6000, 5, 96, 1500, 200, True),          # generic (Di = 96)
    (2, 40000, 8, 64, 20000, 2048, True),       # pool larger than one CTA's shared memory: distributed select
    (2, 20000, 8, 64, 5000, 1500, True),        # <8,64>, ten CTAs a query of 512 entries, the last one ragged (392)
    (1, 9000, 4, 32, 3000, 700, False),         # <4,32>, six CTAs, the last one 440 entries
]


@pytest.mark.parametrize("B,N,Hi,Di,P,k,extreme", REINDEX_CASES)
def test_reindex_paths(B, N, Hi, Di, P, k, extreme, ws, status):
    qi, w, ki = inputs(B * 7 + N + Di, B, 1, N, Hi, Di, extreme)
    q_pos = np.full((B, 1), N - 1, np.int32)
    q_pos[-1, 0] = N // 2 + 1                  # a query part-way through the sequence
    pool, _ = check_full(qi, w, ki, q_pos, min(k, P), P, ws, status)
    qi2, w2, ki2 = inputs(B * 7 + N + Di + 1, B, 1, N, Hi, Di, extreme)
    _, topk = ops.index_topk("REINDEX", dev(q_pos), dev(qi2), w2, dev(ki2), k, pool_in=pool, ws=ws, status=status)
    status.check("reindex")
    rp = pool.cpu().numpy()
    ref = np.stack([[O.index_reindex(qi2[b, 0], w2, ki2[b], rp[b, 0], k)] for b in range(B)])
    got = topk.cpu().numpy()
    assert_list_invariants(got, q_pos, "reindex topk")
    assert_lists_equal(topk, ref, "reindex topk")
    for b in range(B):
        assert set(got[b, 0].tolist()) - {-1} <= set(rp[b, 0].tolist()), "Reindex list outside the pool"


@pytest.mark.parametrize("Hi,Di", [(8, 64), (4, 32), (12, 64)])
def test_reindex_padded_pools(Hi, Di, ws, status):
    """Queries early in their sequences: the Full pools hold fewer valid entries than P
    (-1 after them), and the valid prefix ends inside a CTA's chunk (4 CTAs of 1024
    entries a query), at a chunk's end, or inside the first chunk; one query's prefix is
    shorter than k, so its list ends in -1. Each of the three Reindex scoring forms
    (<8,64>, <4,32>, generic) writes its chunk's positions from its own staging."""
    B, N, P, k = 4, 12000, 4096, 1024
    qi, w, ki = inputs(31 * Hi + Di, B, 1, N, Hi, Di, True)
    q_pos = np.array([[N - 1], [2500], [3071], [700]], np.int32)   # valid pool entries: 4096, 2501, 3072, 701
    pool, _ = check_full(qi, w, ki, q_pos, k, P, ws, status)
    rp = pool.cpu().numpy()
    for b, n_valid in enumerate([4096, 2501, 3072, 701]):
        assert (rp[b, 0, :n_valid] >= 0).all() and (rp[b, 0, n_valid:] == -1).all()
    qi2, w2, ki2 = inputs(31 * Hi + Di + 1, B, 1, N, Hi, Di, True)
    _, topk = ops.index_topk("REINDEX", dev(q_pos), dev(qi2), w2, dev(ki2), k, pool_in=pool, ws=ws, status=status)
    status.check("reindex, padded pools")
    ref = np.stack([[O.index_reindex(qi2[b, 0], w2, ki2[b], rp[b, 0], k)] for b in range(B)])
    got = topk.cpu().numpy()
    assert_list_invariants(got, q_pos, "reindex topk")
    assert_lists_equal(topk, ref, "reindex topk, padded pools")
    assert (got[3, 0, 701:] == -1).all() and (got[3, 0, :701] >= 0).all()


def test_weights_past_the_bound_are_rejected(ws):
    """One weight above the header's bound: the size query returns 0 and the call
    returns CSA2_ERR_RANGE before launching anything."""
    import torch
    from sparse_attention_shared_b200 import capi
    qi, w, ki = inputs(5, 1, 1, 1024, 8, 64, False)
    w = np.ascontiguousarray(w.copy())
    w[3] = max_weight(8, 64) + 1
    topk = torch.empty((1, 1, 16), dtype=torch.int32, device="cuda")
    qp, qid, kid = dev(np.array([[1023]], np.int32)), dev(qi), dev(ki)
    a = ops.make_index_args(capi.CSA2_FULL, qp, qid, w, kid, 16, 0, None, None, topk)
    assert capi.csa2_workspace_bytes(0, a) == 0
    buf = ws.get(1 << 20)
    assert capi.csa2_index_topk(a, buf.data_ptr(), buf.numel(), 0, 0) == 5   # CSA2_ERR_RANGE
    w[3] = max_weight(8, 64)
    assert capi.csa2_workspace_bytes(0, a) > 0


@pytest.mark.parametrize("kind", ["random", "rising", "equal"])
def test_shared_keys_cut(kind, ws, status):
    """Queries that share keys, more of them than SMs: the sampled tiles give each query
    a threshold estimate, the marking pass records its candidates (one bit per
    position), and one CTA per query rescores and cuts them. Random scores and scores
    that rise with the position (runs of equal scores) take the cut; all-equal scores
    make every position a candidate, more than the cut holds, and go to the Full
    kernel's scan and select. Every list bit-exact."""
    from oracle import cpp as C
    B, Tq, N, Hi, Di, k, P = 1, 160, 40000, 8, 64, 512, 2048
    qi, w, ki = inputs(31, B, Tq, N, Hi, Di, False)
    if kind == "rising":
        qi[:] = 1
        ki[:] = (np.arange(N) * 127 // N).astype(np.int8)[None, :, None]
    elif kind == "equal":
        ki[:] = 0
    q_pos = np.broadcast_to(np.arange(N - Tq, N, dtype=np.int32), (B, Tq)).copy()
    pool, topk = ops.index_topk("FULL", dev(q_pos), dev(qi), w, dev(ki), k, P, ws=ws, status=status)
    status.check(kind)
    rpool, rtopk = C.index_full_batch(q_pos, qi, w, ki, k, P)
    assert_list_invariants(topk.cpu().numpy(), q_pos, "topk")
    assert_list_invariants(pool.cpu().numpy(), q_pos, "pool")
    assert_lists_equal(topk, rtopk, f"{kind}: topk")
    assert_lists_equal(pool, rpool, f"{kind}: pool")


@pytest.mark.parametrize("kind", ["random", "rising", "equal"])
def test_full_decode_skewed_scores(kind, ws, status):
    """Decode queries in groups of 12 CTAs with ragged prefixes: random scores, scores that
    rise with the position (every selected entry in the last CTAs' chunks, runs of equal
    scores) and all-equal scores (the whole cut is ties, taken by position). Every list
    bit-exact."""
    from oracle import cpp as C
    B, Tq, N, Hi, Di, k, P = 12, 1, 40000, 8, 64, 512, 2048
    qi, w, ki = inputs(37, B, Tq, N, Hi, Di, False)
    if kind == "rising":
        qi[:] = 1
        ki[:] = (np.arange(N) * 127 // N).astype(np.int8)[None, :, None]
    elif kind == "equal":
        ki[:] = 0
    q_pos = np.full((B, Tq), N - 1, np.int32)
    q_pos[:, 0] -= np.arange(B, dtype=np.int32) * 977   # ragged prefixes
    pool, topk = ops.index_topk("FULL", dev(q_pos), dev(qi), w, dev(ki), k, P, ws=ws, status=status)
    status.check(kind)
    rpool, rtopk = C.index_full_batch(q_pos, qi, w, ki, k, P)
    assert_list_invariants(topk.cpu().numpy(), q_pos, "topk")
    assert_list_invariants(pool.cpu().numpy(), q_pos, "pool")
    assert_lists_equal(topk, rtopk, f"{kind}: topk")
    assert_lists_equal(pool, rpool, f"{kind}: pool")


@pytest.mark.parametrize("kind,Hi,Di", [("random", 8, 64), ("rising", 8, 64), ("equal", 8, 64), ("ragged", 8, 64),
                                        ("random", 4, 32), ("random", 6, 128)])
def test_reindex_one_cta_per_query(kind, Hi, Di, ws, status):
    """Reindex with more queries than SMs: one CTA per query takes its pool as the
    candidate list, rescores the entries on the tensor cores and cuts them in its own
    shared memory. Random scores; scores that rise with the position; all-equal scores
    (the cut is all ties, taken by position); ragged pools padded with -1, some of them
    holding fewer entries than k (the whole pool is the list); 32- and 128-byte keys.
    Every list bit-exact, and every entry taken from the query's pool."""
    from oracle import cpp as C
    if kind == "ragged":
        B, Tq, N, k, P = 2, 80, 3000, 1024, 4096
    elif Di == 64:
        B, Tq, N, k, P = 1, 160, 40000, 2048, 8192
    else:
        B, Tq, N, k, P = 1, 150, 20000, 700, 3000
    qi, w, ki = inputs(41, B, Tq, N, Hi, Di, False)
    qi2, w2, ki2 = inputs(43, B, Tq, N, Hi, Di, False)
    if kind == "rising":
        qi2[:] = 1
        ki2[:] = (np.arange(N) * 127 // N).astype(np.int8)[None, :, None]
    elif kind == "equal":
        ki2[:] = 0
    if kind == "ragged":
        q_pos = np.broadcast_to(np.linspace(200, N - 1, Tq).astype(np.int32), (B, Tq)).copy()
    else:
        q_pos = np.broadcast_to(np.arange(N - Tq, N, dtype=np.int32), (B, Tq)).copy()
    pool, _ = ops.index_topk("FULL", dev(q_pos), dev(qi), w, dev(ki), min(k, P), P, ws=ws, status=status)
    status.check("full")
    _, topk = ops.index_topk("REINDEX", dev(q_pos), dev(qi2), w2, dev(ki2), k, pool_in=pool, ws=ws, status=status)
    status.check(kind)
    rp = pool.cpu().numpy()
    ref = C.index_reindex_batch(qi2, w2, ki2, rp, k)
    got = topk.cpu().numpy()
    assert_list_invariants(got, q_pos, "reindex topk")
    assert_lists_equal(topk, ref, f"{kind}: reindex topk")
    if kind == "ragged":
        assert (got[..., :3] >= 0).all() and (got[..., -1] == -1).any(), "short pools not reached"
    for b in range(B):
        for j in range(Tq):
            assert set(got[b, j].tolist()) - {-1} <= set(rp[b, j].tolist()), "Reindex list outside the pool"
