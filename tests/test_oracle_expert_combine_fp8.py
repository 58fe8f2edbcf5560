"""Pins for the oracle's FP8 expert GEMM followed by combine.

out[t] = sum_k w[t,k] * A[pos[t,k]] @ W_e^T, where A is restored from the
E4M3 codes and 1x128 scales the FP8 dispatch writes and W_e from E4M3 codes
with one scale per 128 x 128 block ("m.nlpx.cn/news/135159" section 4.1;
"lesson14_deepep" section 3).  Checked against things other than its own sum:
  * the E4M3 decoder against PyTorch's float8_e4m3fn cast, all 256 codes;
  * with unit scales the FP8 GEMM is the pinned bf16 expert GEMM of the
    decoded values (every E4M3 value is exact in bf16; decoded by PyTorch);
  * with every code 1.0 the result has a closed form in the block scales
    alone, which fixes which scale belongs to which block (rows and columns
    of the expert matrix, blocks along the inner dimension);
  * row-major and column-major scale layouts give the same result;
  * masked (-1) slots add nothing and a token selection returns its rows.
"""
import numpy as np
import torch

import workloads

ONE = 0x38   # E4M3 code of 1.0


def _setup(T=20, E=4, K=3, seed=3):
    wl = workloads.generate(None, T=T, H=128, E=E, R=2, K=K, A=1, router="topk", seed=seed)
    return wl, wl.topk_idx.numpy(), wl.topk_weights.numpy()


def _codes(rng, shape):
    """Random finite E4M3 codes (no NaN pattern S.1111.111)."""
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    nan = (c & 0x7F) == 0x7F
    c[nan] ^= 0x01
    return c


def _torch_decode_bf16_bits(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.bfloat16)
    return workloads.bf16_bits(t)


def test_e4m3_decoder_all_codes(oracle_lib):
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle_lib.e4m3_value(c) for c in codes])
    nan = np.isnan(want)
    assert nan.sum() == 2 and np.array_equal(nan, np.isnan(got))
    np.testing.assert_array_equal(got[~nan], want[~nan])
    # a few values fixed by the format itself
    assert oracle_lib.e4m3_value(0x7E) == 448.0 and oracle_lib.e4m3_value(0x01) == 2.0 ** -9
    assert oracle_lib.e4m3_value(0x08) == 2.0 ** -6 and oracle_lib.e4m3_value(0xB8) == -1.0


def test_unit_scales_reduce_to_bf16_gemm(oracle_lib):
    wl, idx, tw = _setup()
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    rng = np.random.default_rng(11)
    I, N = 256, 384
    aq = _codes(rng, (L.rows, I))
    wq = _codes(rng, (wl.E, N, I))
    sa = np.ones((L.rows, I // 128), np.float32)
    sw = np.ones((wl.E, N // 128, I // 128), np.float32)
    got = oracle_lib.expert_combine_fp8(aq, sa, wq, sw, idx, L.pos, tw)
    want = oracle_lib.expert_combine(_torch_decode_bf16_bits(aq), _torch_decode_bf16_bits(wq), idx, L.pos, tw)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-300)


def _all_ones_case(oracle_lib, col_major):
    wl, idx, tw = _setup(T=16, K=2, seed=21)
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    rng = np.random.default_rng(12)
    I, N = 384, 256                       # 3 inner blocks, 2 column blocks: a transposed index shows
    IB, NB = I // 128, N // 128
    aq = np.full((L.rows, I), ONE, np.uint8)
    wq = np.full((wl.E, N, I), ONE, np.uint8)
    sa = rng.uniform(0.5, 2.0, (L.rows, IB)).astype(np.float32)
    sw = rng.uniform(0.5, 2.0, (wl.E, NB, IB)).astype(np.float32)
    if col_major:
        ld = L.rows + 3
        buf = np.full(IB * ld, np.nan, np.float32)   # the gap past the rows is never read
        for b in range(IB):
            buf[b * ld:b * ld + L.rows] = sa[:, b]
        got = oracle_lib.expert_combine_fp8(aq, buf, wq, sw, idx, L.pos, tw, scale_ld=ld)
    else:
        got = oracle_lib.expert_combine_fp8(aq, sa, wq, sw, idx, L.pos, tw)
    # with all codes 1.0, block (b) of row r dotted with block (b) of W_e row n is 128 * sa * sw
    want = np.zeros((wl.T, N))
    for t in range(wl.T):
        for k in range(wl.K):
            e, r = idx[t, k], L.pos[t, k]
            for n in range(N):
                want[t, n] += float(tw[t, k]) * sum(
                    128.0 * float(sa[r, b]) * float(sw[e, n // 128, b]) for b in range(IB))
    np.testing.assert_allclose(got, want, rtol=1e-12)
    return got


def test_block_scales_closed_form(oracle_lib):
    _all_ones_case(oracle_lib, col_major=False)


def test_column_major_scales(oracle_lib):
    np.testing.assert_array_equal(_all_ones_case(oracle_lib, col_major=True),
                                  _all_ones_case(oracle_lib, col_major=False))


def test_masked_slots_and_selection_fp8(oracle_lib):
    wl, idx, tw = _setup(T=12, K=3, seed=14)
    idx = idx.copy()
    idx[::4, 2] = -1
    L = oracle_lib.layout(idx, wl.E, wl.R, wl.A)
    rng = np.random.default_rng(15)
    I, N = 128, 128
    aq = _codes(rng, (max(L.rows, 1), I))
    wq = _codes(rng, (wl.E, N, I))
    sa = rng.uniform(0.01, 0.1, (max(L.rows, 1), 1)).astype(np.float32)
    sw = rng.uniform(0.01, 0.1, (wl.E, 1, 1)).astype(np.float32)
    full = oracle_lib.expert_combine_fp8(aq, sa, wq, sw, idx, L.pos, tw)
    tw0 = tw.copy()
    tw0[idx < 0] = 0.0
    np.testing.assert_allclose(full, oracle_lib.expert_combine_fp8(aq, sa, wq, sw, idx, L.pos, tw0), rtol=1e-12)
    sel = np.array([3, 0, 11], np.int32)
    np.testing.assert_array_equal(oracle_lib.expert_combine_fp8(aq, sa, wq, sw, idx, L.pos, tw, sel_tokens=sel),
                                  full[sel])
