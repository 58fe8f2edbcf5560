"""Pins for the oracle's expert GEMM followed by combine.

out[t] = sum_k w[t,k] * act[pos[t,k]] @ W_e^T with e = topk_idx[t,k]
("lesson14_deepep" practice task: experts transform the rows they received,
combine adds weight * expert output back per token).  Checked against closed
forms that do not restate the sum:
  * scaled-identity experts W_e = c_e * I reduce it to the pinned combine of
    the rows scaled by c_e;
  * rank-1 experts W_e = u_e v_e^T give sum_k w * (act . v_e) * u_e;
  * masked (-1) slots add nothing.
"""
import numpy as np

import workloads


def _bf16(a):
    import torch
    return workloads.bf16_bits(torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16))


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _setup(T=24, I=32, E=4, K=3, seed=3):
    wl = workloads.generate(None, T=T, H=I, E=E, R=2, K=K, A=1, router="topk", seed=seed)
    return wl, wl.topk_idx.numpy(), wl.topk_weights.numpy()


def test_scaled_identity_experts(oracle_lib):
    wl, idx, tw = _setup()
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    rng = np.random.default_rng(4)
    act = _bf16(rng.standard_normal((L.rows, 32)))
    c = np.array([1.0, -2.0, 0.5, 4.0])                    # exact in bf16
    w = _bf16(c[:, None, None] * np.eye(32)[None])          # [E, N=I, I]
    got = oracle_lib.expert_combine(act, w, idx, L.pos, tw)
    # the same as combining the rows scaled by their expert's c_e
    expert_of_row = np.searchsorted(L.expert_offsets, np.arange(L.rows), side="right") - 1
    scaled = _bf16(_f64(act) * c[expert_of_row][:, None])
    want = oracle_lib.combine(scaled, L.pos, tw)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_rank_one_experts(oracle_lib):
    wl, idx, tw = _setup(T=20, K=2, seed=9)
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    rng = np.random.default_rng(5)
    I, N = 32, 48
    act = _bf16(rng.standard_normal((L.rows, I)))
    u = np.round(rng.standard_normal((wl.E, N)) * 4) / 4   # few bits: products exact in bf16
    v = np.round(rng.standard_normal((wl.E, I)) * 4) / 4
    w = _bf16(u[:, :, None] * v[:, None, :])                # W_e[n, i] = u_e[n] v_e[i]
    got = oracle_lib.expert_combine(act, w, idx, L.pos, tw)
    a = _f64(act)
    want = np.zeros((wl.T, N))
    for t in range(wl.T):
        for k in range(wl.K):
            e, r = idx[t, k], L.pos[t, k]
            want[t] += float(tw[t, k]) * float(a[r] @ v[e]) * u[e]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_masked_slots_and_selection(oracle_lib):
    wl, idx, tw = _setup(T=16, K=3, seed=12)
    idx = idx.copy()
    idx[::3, 1] = -1
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    rng = np.random.default_rng(6)
    act = _bf16(rng.standard_normal((max(L.rows, 1), 32)))
    w = _bf16(rng.standard_normal((wl.E, 16, 32)))
    full = oracle_lib.expert_combine(act, w, idx, L.pos, tw)
    tw0 = tw.copy()
    tw0[idx < 0] = 0.0
    np.testing.assert_allclose(full, oracle_lib.expert_combine(act, w, idx, L.pos, tw0), rtol=1e-12)
    sel = np.array([5, 0, 15], np.int32)
    np.testing.assert_array_equal(oracle_lib.expert_combine(act, w, idx, L.pos, tw, sel), full[sel])
