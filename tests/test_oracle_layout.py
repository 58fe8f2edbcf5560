"""Pins for the oracle's layout (counts, offsets, stable permutation).

The oracle is checked against things other than itself:
  * the worked example of the lesson14_deepep practice task (golden fixture);
  * a second, sort-based definition over every routing table of tiny sizes;
  * invariants that any correct layout satisfies, on the five workloads.
"""
import itertools
import json
import os

import numpy as np
import pytest

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p3_worked_example.json")


def test_worked_example(oracle_lib):
    g = json.load(open(GOLDEN))
    idx = np.array(g["topk_idx"], dtype=np.int64)
    assert idx.shape == (g["num_tokens"], g["num_topk"])
    for case in g["cases"]:
        L = oracle_lib.layout(idx, g["num_experts"], case["num_ranks"], case["expert_alignment"])
        assert L.status == 0
        assert int(L.num_tokens_per_expert.sum()) == g["conservation_total"]
        for key in ("num_tokens_per_expert", "num_tokens_per_rank", "is_token_in_rank",
                    "expert_offsets", "rank_offsets", "pos", "row_src", "row_slot"):
            np.testing.assert_array_equal(getattr(L, key), np.array(case[key]), err_msg=key)
        # each expert's real rows are its queue from the page's loop, in order
        for e, queue in g["queues"].items():
            e = int(e)
            start = L.expert_offsets[e]
            got = [(int(L.row_src[r]), int(L.row_slot[r]))
                   for r in range(start, start + L.num_tokens_per_expert[e])]
            assert got == [tuple(q) for q in queue]


def naive_layout(idx, E, R, A):
    """Second definition: sort the (expert, token, k) triples, pad each segment."""
    T, K = idx.shape
    Lr = E // R
    # -1 marks an unused slot: no row, pos = -1
    triples = sorted((int(idx[t, k]), t, k) for t in range(T) for k in range(K) if idx[t, k] != -1)
    rows, offsets, pos = [], [0], {}
    for e in range(E):
        seg = [(t, k) for (ee, t, k) in triples if ee == e]
        for tk in seg:
            pos[tk] = len(rows)
            rows.append(tk)
        rows.extend([None] * ((-len(seg)) % A))
        offsets.append(len(rows))
    counts = [sum(1 for tr in triples if tr[0] == e) for e in range(E)]
    ranks_of = [set(int(idx[t, k]) // Lr for k in range(K) if idx[t, k] != -1) for t in range(T)]
    in_rank = [[1 if r in ranks_of[t] else 0 for r in range(R)] for t in range(T)]
    per_rank = [sum(in_rank[t][r] for t in range(T)) for r in range(R)]
    return dict(
        num_tokens_per_expert=counts, num_tokens_per_rank=per_rank,
        is_token_in_rank=np.array(in_rank, dtype=np.uint8).reshape(T, R),
        expert_offsets=offsets, rank_offsets=[offsets[r * Lr] for r in range(R + 1)],
        pos=np.array([[pos.get((t, k), -1) for k in range(K)] for t in range(T)], dtype=np.int32).reshape(T, K),
        row_src=[-1 if x is None else x[0] for x in rows],
        row_slot=[-1 if x is None else x[1] for x in rows])


def _divisors(n):
    return [d for d in range(1, n + 1) if n % d == 0]


def test_bruteforce_tiny(oracle_lib):
    n_cases = 0
    for T in range(0, 4):
        for E in range(1, 5):
            for K in (1, 2):
                if T * K > 6:
                    continue
                tables = itertools.product(range(-1 if E <= 3 else 0, E), repeat=T * K)
                for flat in tables:
                    idx = np.array(flat, dtype=np.int64).reshape(T, K)
                    for R in _divisors(E):
                        for A in (1, 2, 3):
                            L = oracle_lib.layout(idx, E, R, A)
                            ref = naive_layout(idx, E, R, A)
                            assert L.status == 0
                            for key, val in ref.items():
                                np.testing.assert_array_equal(
                                    getattr(L, key), np.asarray(val).reshape(getattr(L, key).shape),
                                    err_msg=f"{key} T={T} E={E} K={K} R={R} A={A} idx={flat}")
                            n_cases += 1
    assert n_cases > 10000


def check_layout_invariants(L, idx, E, R, A, w=None):
    T, K = idx.shape
    Lr = E // R
    cnt = L.num_tokens_per_expert
    assert int(cnt.sum()) == T * K                       # conservation (no masked slots here)
    np.testing.assert_array_equal(cnt, np.bincount(idx.ravel(), minlength=E))
    pad = -(-cnt // A) * A
    np.testing.assert_array_equal(np.diff(L.expert_offsets), pad)
    assert L.expert_offsets[0] == 0 and L.rows == int(pad.sum())
    assert L.rows <= L.capacity
    np.testing.assert_array_equal(L.rank_offsets, L.expert_offsets[::Lr])
    # pos is a bijection onto the non-padding rows, inverse of (row_src, row_slot)
    flat = L.pos.ravel()
    assert len(np.unique(flat)) == T * K
    tt, kk = np.divmod(np.arange(T * K), K)
    np.testing.assert_array_equal(L.row_src[flat], tt)
    np.testing.assert_array_equal(L.row_slot[flat], kk)
    real = np.zeros(L.rows, bool)
    real[flat] = True
    assert (L.row_src[~real] == -1).all() and (L.row_slot[~real] == -1).all()
    # every row lies in the segment of its expert; segments are (t, k)-sorted
    seg_of_row = np.searchsorted(L.expert_offsets, np.arange(L.rows), side="right") - 1
    np.testing.assert_array_equal(seg_of_row[flat], idx.ravel())
    for e in range(E):
        a, b = L.expert_offsets[e], L.expert_offsets[e] + cnt[e]
        key = L.row_src[a:b].astype(np.int64) * K + L.row_slot[a:b]
        assert (np.diff(key) > 0).all()
        assert (L.row_src[b:L.expert_offsets[e + 1]] == -1).all()
    # rank membership and distinct-token counts
    member = np.zeros((T, R), np.uint8)
    member[np.repeat(np.arange(T), K), (idx // Lr).ravel()] = 1
    np.testing.assert_array_equal(L.is_token_in_rank, member)
    np.testing.assert_array_equal(L.num_tokens_per_rank, member.sum(0))
    if w is not None:
        np.testing.assert_array_equal(L.row_weight[flat], w.ravel())
        assert (L.row_weight[~real] == 0).all()


@pytest.mark.parametrize("name", list(workloads.CONFIGS))
def test_invariants_on_workloads(oracle_lib, name):
    wl = workloads.generate(name, with_x=False)
    idx, w = wl.topk_idx.numpy(), wl.topk_weights.numpy()
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A, topk_weights=w)
    assert L.status == 0
    check_layout_invariants(L, idx, wl.E, wl.R, wl.A, w)


def test_workload_shapes():
    wl = workloads.generate("tiny")
    assert wl.x.shape == (64, 256) and wl.topk_idx.shape == (64, 2)
    idx = wl.topk_idx.numpy()
    assert (idx[:, 0] != idx[:, 1]).all()                 # distinct experts
    np.testing.assert_allclose(wl.topk_weights.numpy().sum(1), 1.0, rtol=1e-6)
    d = workloads.generate("dsv3", with_x=False).topk_idx.numpy()
    groups = d // 32
    assert all(len(set(g)) <= 4 for g in groups)          # group-limited: at most 4 groups
    assert all(len(set(r)) == 8 for r in d)               # 8 distinct experts


def test_invalid_expert_ids(oracle_lib):
    idx = np.array([[0, 1], [2, 4]], dtype=np.int64)
    assert oracle_lib.layout(idx, 4, 2, 1).status == oracle_lib.BAD_EXPERT
    idx = np.array([[0, -2]], dtype=np.int64)
    assert oracle_lib.layout(idx, 4, 2, 1).status == oracle_lib.BAD_EXPERT
    assert oracle_lib.layout(np.zeros((1, 1), np.int64), 4, 3, 1).status == oracle_lib.BAD_ARG


def test_masked_slots(oracle_lib):
    """-1 marks an unused top-k slot: no row, not counted, pos = -1."""
    idx = np.array([[0, -1], [-1, -1], [3, 0]], dtype=np.int64)
    L = oracle_lib.layout(idx, 4, 2, 2)
    assert L.status == 0
    assert list(L.num_tokens_per_expert) == [2, 0, 0, 1]
    assert L.pos.tolist() == [[0, -1], [-1, -1], [2, 1]]
    assert list(L.expert_offsets) == [0, 2, 2, 2, 4]
    assert list(L.row_src) == [0, 2, 2, -1]
    assert L.is_token_in_rank.tolist() == [[1, 0], [0, 0], [1, 1]]
    assert list(L.num_tokens_per_rank) == [2, 1]


def test_empty_and_degenerate(oracle_lib):
    L = oracle_lib.layout(np.zeros((0, 4), np.int64), 8, 2, 4)
    assert L.status == 0 and L.rows == 0
    np.testing.assert_array_equal(L.expert_offsets, np.zeros(9))
    # every token to one expert
    idx = np.full((5, 1), 3, np.int64)
    L = oracle_lib.layout(idx, 4, 4, 4)
    assert list(L.expert_offsets) == [0, 0, 0, 0, 8]
    assert list(L.pos.ravel()) == [0, 1, 2, 3, 4]
    assert list(L.row_src) == [0, 1, 2, 3, 4, -1, -1, -1]
