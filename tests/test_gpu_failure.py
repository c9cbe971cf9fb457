"""Failure detection of the indexer's inter-CTA waits, without a GPU fault.

The CTAs that select one query's lists meet at group barriers (spins on a counter
in the workspace). Here the host sets a short wait budget and injects a fault on
the host side: the last CTA of each group leaves before its first barrier, so the
other CTAs' waits run out. The call must end promptly, report CSA2_ERR_TIMEOUT in
the status word, and leave the device usable: after the workspace is zeroed again,
the next call gives the oracle's lists."""
import time

import numpy as np
import pytest

import synth
from oracle import csa2_oracle as O
from sparse_attention_shared_b200 import capi, ops

from gpu_util import assert_lists_equal, dev

pytestmark = pytest.mark.gpu

CSA2_ERR_TIMEOUT = 8
SHORT_BUDGET = 20000        # SM cycles: about 10 us at the boost clock


def _inputs(seed, B, N):
    qi = synth.randint_i8(seed, 1, (B, 1, 8, 64))
    ki = synth.randint_i8(seed, 2, (B, N, 64))
    w = synth.randint_i32(seed, 3, (8,), 1, 8)
    q_pos = np.full((B, 1), N - 1, np.int32)
    return qi, w, ki, q_pos


def _timed_failing_call(fn):
    capi.check(capi.csa2_set_wait_controls(SHORT_BUDGET, 1), "wait controls")
    try:
        t0 = time.perf_counter()
        fn()
        import torch
        torch.cuda.synchronize()
        return time.perf_counter() - t0
    finally:
        capi.check(capi.csa2_set_wait_controls(0, 0), "wait controls")


@pytest.mark.parametrize("mode", ["FULL", "REINDEX"])
def test_group_wait_runs_out_and_the_next_call_is_exact(mode):
    # Groups of several CTAs per query, which meet at spin barriers: 4 queries x 400000
    # keys in Full mode, and a Reindex pool of 20000 entries (the group's distributed select).
    B, N, k, P = 4, 400000, 1024, 20000
    qi, w, ki, q_pos = _inputs(11, B, N)
    ws, st = ops.Workspace(), ops.Status()
    dq, dqi, dki = dev(q_pos), dev(qi), dev(ki)
    pool, _ = ops.index_topk("FULL", dq, dqi, w, dki, k, P, ws=ws, status=st)   # warm: library, attributes
    st.check("warm-up")
    if mode == "FULL":
        call = lambda: ops.index_topk("FULL", dq, dqi, w, dki, k, P, ws=ws, status=st)
    else:
        call = lambda: ops.index_topk("REINDEX", dq, dqi, w, dki, k, pool_in=pool, ws=ws, status=st)
    elapsed = _timed_failing_call(call)
    code, detail = st.read()
    assert code == CSA2_ERR_TIMEOUT, f"status {code} (detail {detail})"
    assert elapsed < 0.5, f"the failing call took {elapsed:.3f} s"
    # recovery: zero the workspace and the status, then an exact call
    ws.reset()
    st.clear()
    rp = pool.cpu().numpy()
    if mode == "FULL":
        p2, t2 = ops.index_topk("FULL", dq, dqi, w, dki, k, P, ws=ws, status=st)
        st.check("after recovery")
        for b in range(B):
            rpool, rtopk = O.index_full(qi[b, 0], w, ki[b], N - 1, k, P)
            assert_lists_equal(t2[b, 0], rtopk, "topk after recovery")
            assert_lists_equal(p2[b, 0], rpool, "pool after recovery")
    else:
        _, t2 = ops.index_topk("REINDEX", dq, dqi, w, dki, k, pool_in=pool, ws=ws, status=st)
        st.check("after recovery")
        for b in range(B):
            assert_lists_equal(t2[b, 0], O.index_reindex(qi[b, 0], w, ki[b], rp[b, 0], k), "reindex after recovery")
