"""Pins for the oracle's dispatch (bf16, FP8) and combine.

  * identity experts: combine(dispatch(x)) == x * sum_k w (round-trip check
    recommended on the 2kiu.com page, section 3.3);
  * one-hot weights with per-expert marker rows pick the row of the right
    expert for the right token;
  * the lesson14_deepep practice task, restated: per-expert linear maps on the
    dispatched rows, combined, equal the dense per-token reference
    sum_k w * (x W_e);
  * FP8: error bound of E4M3 rounding, the block maximum lands on +-448, all
    K copies are identical bytes, padding rows are zero.
"""
import numpy as np
import pytest
import torch

import workloads


def _setup(T=48, H=256, E=8, R=4, K=3, A=4, seed=11, router="uniform"):
    wl = workloads.generate(None, T=T, H=H, E=E, R=R, K=K, A=A, router=router, seed=seed)
    return wl, wl.topk_idx.numpy(), wl.topk_weights.numpy(), workloads.bf16_bits(wl.x)


def _to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _to_bf16_bits(a):
    return workloads.bf16_bits(torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16))


@pytest.mark.parametrize("A", [1, 4])
def test_identity_round_trip(oracle_lib, A):
    wl, idx, w, xb = _setup(A=A)
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A, topk_weights=w)
    recv = oracle_lib.dispatch_bf16(xb, L.row_src)
    assert recv.shape == (L.rows, wl.H)
    pad = L.row_src < 0
    assert (recv[pad] == 0).all()
    out = oracle_lib.combine(recv, L.pos, w)
    want = _to_f64(xb) * w.astype(np.float64).sum(1, keepdims=True)
    np.testing.assert_allclose(out, want, rtol=1e-13, atol=1e-13)


def test_one_hot_selects_expert_row(oracle_lib):
    wl, idx, w, xb = _setup(T=40, E=16, R=4, K=4, A=3)
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    expert_of_row = np.searchsorted(L.expert_offsets, np.arange(L.rows), side="right") - 1
    # y row = x row + marker, marker = 4*expert + slot (small integers, exact in bf16 for |x|<2)
    recv = oracle_lib.dispatch_bf16(xb, L.row_src)
    marker = (4 * expert_of_row + np.maximum(L.row_slot, 0)).astype(np.float64)
    y = np.zeros((L.rows, wl.H), np.float64) + marker[:, None]
    yb = _to_bf16_bits(y)
    for kstar in range(wl.K):
        oh = np.zeros_like(w)
        oh[:, kstar] = 1.0
        out = oracle_lib.combine(yb, L.pos, oh)
        want = 4 * idx[:, kstar] + kstar
        np.testing.assert_array_equal(out, np.repeat(want[:, None], wl.H, 1).astype(np.float64))
    # and the dispatched rows carry the right token
    np.testing.assert_array_equal(recv[L.pos.ravel()], np.repeat(xb, wl.K, axis=0))


def test_lesson_exercise_restated(oracle_lib):
    rng = np.random.default_rng(1234)
    wl, idx, w, xb = _setup(T=32, H=128, E=8, R=2, K=2, A=1, seed=5)
    x = _to_f64(xb)
    W = rng.standard_normal((wl.E, wl.H, wl.H)) / np.sqrt(wl.H)
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    recv = _to_f64(oracle_lib.dispatch_bf16(xb, L.row_src))
    expert_of_row = np.searchsorted(L.expert_offsets, np.arange(L.rows), side="right") - 1
    y = np.einsum("rh,rhg->rg", recv, W[expert_of_row])
    yb = _to_bf16_bits(y)
    out = oracle_lib.combine(yb, L.pos, w)
    dense = np.zeros((wl.T, wl.H))
    for k in range(wl.K):
        dense += w[:, k:k + 1].astype(np.float64) * np.einsum("th,thg->tg", x, W[idx[:, k]])
    # y was rounded to bf16: error <= sum_k |w| * |y| * 2^-8
    bound = sum(np.abs(w[:, k:k + 1]) * np.abs(y[L.pos[:, k]]) for k in range(wl.K)) * 2.0 ** -8
    assert (np.abs(out - dense) <= bound + 1e-12).all()


def e4m3_decode_array(codes):
    c = codes.astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    v = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    return s * v


@pytest.mark.parametrize("A", [1, 5])
def test_fp8_dispatch_properties(oracle_lib, A):
    wl, idx, w, xb = _setup(T=36, H=512, E=8, R=2, K=4, A=A, seed=3)
    # add a zero block, a tiny block and a large-range block
    x = _to_f64(xb)
    x[0, :128] = 0.0
    x[1, 128:256] *= 1e-6
    x[2, 256:384] *= 300.0
    xb = _to_bf16_bits(x)
    x = _to_f64(xb)
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    q, s = oracle_lib.dispatch_fp8(xb, L.row_src)
    pad = L.row_src < 0
    assert (q[pad] == 0).all() and (s[pad] == 0).all()
    # K copies of a token are byte-identical
    for t in range(wl.T):
        rows = L.pos[t]
        assert (q[rows] == q[rows[0]]).all() and (s[rows] == s[rows[0]]).all()
    real = np.flatnonzero(~pad)
    xr = x[L.row_src[real]].reshape(len(real), -1, 128)
    qv = e4m3_decode_array(q[real]).reshape(len(real), -1, 128)
    sc = s[real].astype(np.float64)[:, :, None]
    amax = np.abs(xr).max(axis=2, keepdims=True)
    big = amax[..., 0] >= 1e-4
    # the block maximum maps onto +-448 exactly
    assert (np.abs(qv).max(axis=2)[big] == 448.0).all()
    # dequantised scale times 448 reproduces amax to fp32 rounding
    np.testing.assert_allclose((sc[..., 0] * 448.0)[big], amax[..., 0][big], rtol=2e-7)
    # E4M3 rounding: relative 2^-4 in the normal range, 2^-10 * scale below 2^-6
    err = np.abs(xr - qv * sc)
    assert (err <= np.abs(xr) * 2.0 ** -4 * (1 + 1e-6) + sc * 2.0 ** -10 * (1 + 1e-6)).all()
    # the all-zero block encodes to zero codes
    t0_rows = L.pos[0]
    assert (q[t0_rows, :128] == 0).all()


def test_selected_rows_and_tokens(oracle_lib):
    wl, idx, w, xb = _setup(T=30, H=256, E=8, R=2, K=2, A=2, seed=9)
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    full = oracle_lib.dispatch_bf16(xb, L.row_src)
    sel = np.array([L.rows - 1, 0, 5, 3], np.int32)
    np.testing.assert_array_equal(oracle_lib.dispatch_bf16(xb, L.row_src, sel), full[sel])
    qf, sf = oracle_lib.dispatch_fp8(xb, L.row_src)
    qs, ss = oracle_lib.dispatch_fp8(xb, L.row_src, sel)
    np.testing.assert_array_equal(qs, qf[sel])
    np.testing.assert_array_equal(ss, sf[sel])
    out = oracle_lib.combine(full, L.pos, w)
    tsel = np.array([7, 0, 29], np.int32)
    np.testing.assert_array_equal(oracle_lib.combine(full, L.pos, w, tsel), out[tsel])


def test_masked_slots_round_trip(oracle_lib):
    """Identity experts with some slots masked (-1): out = x * sum of the unmasked weights."""
    wl, idx, w, xb = _setup(T=40, H=256, E=8, R=2, K=4, A=3, seed=17)
    rng = np.random.default_rng(3)
    idx = idx.copy()
    idx[rng.random(idx.shape) < 0.3] = -1
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A, topk_weights=w)
    assert L.status == 0
    assert int(L.num_tokens_per_expert.sum()) == int((idx >= 0).sum())
    assert (L.pos[idx < 0] == -1).all()
    recv = oracle_lib.dispatch_bf16(xb, L.row_src)
    out = oracle_lib.combine(recv, L.pos, w)
    wsum = np.where(idx >= 0, w.astype(np.float64), 0.0).sum(1, keepdims=True)
    np.testing.assert_allclose(out, _to_f64(xb) * wsum, rtol=1e-13, atol=1e-13)
