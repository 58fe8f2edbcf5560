"""Pins for the oracle's low-latency (static, masked) layout.

Every expert owns M fixed received rows e*M .. e*M+M-1; its pairs fill them
in (token, k) order and recv_count[e] is the mask ("lesson14_deepep" section
2(1) and the low_latency_dispatch listing of section 3).  Checked against:
  * the worked example of the lesson14_deepep practice task (golden fixture:
    each expert's queue, in the page's loop order, becomes its slots);
  * the sort-based second definition of the normal layout in
    test_oracle_layout.py, re-offset to e*M, over every tiny routing table;
  * identity experts: combine(dispatch(x)) = x * the weights of kept pairs.
"""
import itertools
import json

import numpy as np

import workloads
from test_oracle_layout import GOLDEN, naive_layout


def test_ll_worked_example(oracle_lib):
    g = json.load(open(GOLDEN))
    idx = np.array(g["topk_idx"], dtype=np.int64)
    E = g["num_experts"]
    for M in (g["num_tokens"], 7, 1):
        L = oracle_lib.ll_layout(idx, E, M)
        want_pos = np.full(idx.shape, -1, np.int32)
        want_cnt = np.zeros(E, np.int32)
        dropped = False
        for e, queue in g["queues"].items():
            e = int(e)
            for j, (t, k) in enumerate(queue):
                if j < M:
                    want_pos[t, k] = e * M + j
                else:
                    dropped = True
            want_cnt[e] = min(len(queue), M)
        assert L.status == (oracle_lib.SLOT_OVERFLOW if dropped else oracle_lib.OK)
        np.testing.assert_array_equal(L.pos, want_pos)
        np.testing.assert_array_equal(L.recv_count, want_cnt)


def expected_ll(idx, E, M):
    """Re-offset the sort-based normal layout (A = 1) to fixed slots e*M."""
    ref = naive_layout(idx, E, 1, 1)
    off = np.asarray(ref["expert_offsets"])
    pos = np.asarray(ref["pos"]).reshape(idx.shape)
    out = np.full(idx.shape, -1, np.int32)
    for (t, k), p in np.ndenumerate(pos):
        if p >= 0:
            e = int(idx[t, k])
            j = p - off[e]
            out[t, k] = e * M + j if j < M else -1
    cnt = np.minimum(np.asarray(ref["num_tokens_per_expert"]), M).astype(np.int32)
    overflow = bool((np.asarray(ref["num_tokens_per_expert"]) > M).any())
    return out, cnt, overflow


def test_ll_bruteforce_tiny(oracle_lib):
    n = 0
    for T in range(0, 4):
        for E in (1, 2, 3):
            for K in (1, 2):
                if T * K > 6:
                    continue
                for flat in itertools.product(range(-1, E), repeat=T * K):
                    idx = np.array(flat, dtype=np.int64).reshape(T, K)
                    for M in (1, 2, 3, 6):
                        L = oracle_lib.ll_layout(idx, E, M)
                        pos, cnt, overflow = expected_ll(idx, E, M)
                        assert L.status == (oracle_lib.SLOT_OVERFLOW if overflow else oracle_lib.OK)
                        np.testing.assert_array_equal(L.pos, pos, err_msg=f"T={T} E={E} K={K} M={M} {flat}")
                        np.testing.assert_array_equal(L.recv_count, cnt)
                        n += 1
    assert n > 5000


def test_ll_round_trip(oracle_lib):
    wl = workloads.generate(None, T=40, H=256, E=8, R=2, K=4, A=1, router="topk", seed=19)
    idx, w, xb = wl.topk_idx.numpy().copy(), wl.topk_weights.numpy(), workloads.bf16_bits(wl.x)
    idx[np.random.default_rng(2).random(idx.shape) < 0.2] = -1
    M = 40
    L = oracle_lib.ll_layout(idx, wl.E, M)
    assert L.status == oracle_lib.OK
    assert int(L.recv_count.sum()) == int((idx >= 0).sum())
    recv = oracle_lib.dispatch_bf16(xb, L.row_src)
    out = oracle_lib.combine(recv, L.pos, w)
    wsum = np.where(idx >= 0, w.astype(np.float64), 0.0).sum(1, keepdims=True)
    x = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    np.testing.assert_allclose(out, x * wsum, rtol=1e-13, atol=1e-13)
    # every used slot of expert e lies in [e*M, e*M + recv_count[e])
    used = L.pos[L.pos >= 0]
    e_of = used // M
    assert ((used - e_of * M) < L.recv_count[e_of]).all()
    assert len(np.unique(used)) == len(used)


def test_ll_invalid_ids(oracle_lib):
    assert oracle_lib.ll_layout(np.array([[0, 4]], np.int64), 4, 2).status == oracle_lib.BAD_EXPERT
    assert oracle_lib.ll_layout(np.array([[-3, 0]], np.int64), 4, 2).status == oracle_lib.BAD_EXPERT
    L = oracle_lib.ll_layout(np.zeros((0, 3), np.int64), 4, 2)
    assert L.status == oracle_lib.OK and not L.recv_count.any()
