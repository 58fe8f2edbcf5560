"""Parity of the FP8 expert GEMM + fused combine (ep_expert_combine_fp8) with the oracle.

out[t] = bf16(sum_k w[t,k] * A[pos[t,k]] @ W_e^T) with A and W_e restored from
E4M3 codes and block scales (1x128 per row, 128x128 per expert matrix);
compared with the oracle's fp64 sum within rtol 1e-2 / atol 1e-3 (E4M3
products summed in fp32 per 128-deep block, scaled and summed in fp32,
fp32 atomic adds, bf16 output).  The rows come either from seeded codes
or from the FP8 dispatch itself (the oracle then takes its own dispatch's
codes, which the dispatch parity tests show to be the same bytes).
"""
import numpy as np
import pytest
import torch

import combine_ep_get_08_b200 as ep
import oracle
import workloads
from ep_harness import combine_close, gpu_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_ep_get_08_b200 import build_lib
    build_lib.build()
    oracle.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def codes(rng, shape, emin=4, emax=10):
    """Seeded E4M3 codes with random sign and mantissa, exponent field in [emin, emax]
    (values between 2^-3 and 2^3.9)."""
    sign = rng.integers(0, 2, size=shape, dtype=np.uint8) << 7
    exp = rng.integers(emin, emax + 1, size=shape, dtype=np.uint8) << 3
    man = rng.integers(0, 8, size=shape, dtype=np.uint8)
    return sign | exp | man


def expert_weights(rng, E, N, I):
    wq = codes(rng, (E, N, I))
    ws = (rng.uniform(0.5, 1.5, (E, N // 128, I // 128)) / np.sqrt(I)).astype(np.float32)
    return wq, ws


def run_gemm(g, wl, aq_d, sa_d, I, wq, ws, N):
    dev = torch.device("cuda")
    tw = wl.topk_weights.to(dev)
    acc = torch.full((wl.T, N), 7.0, dtype=torch.float32, device=dev)
    out = torch.empty((wl.T, N), dtype=torch.bfloat16, device=dev)
    ep.ep_expert_combine_fp8(g.handle, aq_d, sa_d, I, torch.from_numpy(wq).to(dev), torch.from_numpy(ws).to(dev),
                             N, tw, acc, out)
    torch.cuda.synchronize()
    assert ep.ep_get_status(g.handle) == 0
    return out


def run_case(wl, I, N, idx=None, check_tokens=None, seed=3, col_major=False):
    dev = torch.device("cuda")
    if idx is not None:
        wl.topk_idx = idx
    g = gpu_layout(wl)
    try:
        assert g.status == 0
        rng = np.random.default_rng(seed)
        IB = I // 128
        aq = codes(rng, (g.cap, I))
        sa = rng.uniform(0.25, 1.0, (g.cap, IB)).astype(np.float32)
        if col_major:
            ep.ep_set_scale_layout(g.handle, ep.EP_SCALES_COL_MAJOR_TMA)
            ld = (g.cap + 3) // 4 * 4
            sa_buf = np.full(IB * ld, np.nan, np.float32)   # the gap past the rows is never read
            for b in range(IB):
                sa_buf[b * ld:b * ld + g.cap] = sa[:, b]
        else:
            ld, sa_buf = 0, sa
        wq, ws = expert_weights(rng, wl.E, N, I)
        out = run_gemm(g, wl, torch.from_numpy(aq).to(dev), torch.from_numpy(sa_buf).to(dev), I, wq, ws, N)
        o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A)
        sel = None if check_tokens is None else np.asarray(check_tokens, np.int32)
        rows = max(g.rows, 1)
        if col_major:
            ref = oracle.expert_combine_fp8(aq[:rows], sa_buf, wq, ws, wl.topk_idx.numpy(), o.pos,
                                            wl.topk_weights.numpy(), scale_ld=ld, sel_tokens=sel)
        else:
            ref = oracle.expert_combine_fp8(aq[:rows], sa[:rows], wq, ws, wl.topk_idx.numpy(), o.pos,
                                            wl.topk_weights.numpy(), sel_tokens=sel)
        got = out if sel is None else out[torch.from_numpy(sel).long().to(dev)]
        combine_close(got, ref)
        return out
    finally:
        ep.ep_handle_destroy(g.handle)


def test_small_one_tile_column():
    wl = workloads.generate(None, T=256, H=128, E=8, R=2, K=4, A=128, router="topk", seed=81)
    run_case(wl, I=128, N=256)


def test_many_tiles_persistent():
    """More tiles than SMs, 4 k-blocks per tile: the ring and both TMEM partial
    buffers are reused many times."""
    wl = workloads.generate(None, T=2048, H=128, E=16, R=4, K=8, A=128, router="topk", seed=82)
    run_case(wl, I=512, N=1024, check_tokens=np.r_[0:48, 2000:2048])


def test_masked_slots_and_skew():
    wl = workloads.generate(None, T=512, H=128, E=32, R=8, K=6, A=256, router="zipf", seed=83)
    idx = wl.topk_idx.clone()
    idx[torch.rand(idx.shape, generator=torch.Generator().manual_seed(3)) < 0.2] = -1
    run_case(wl, I=256, N=512, idx=idx)


def test_column_major_scales():
    wl = workloads.generate(None, T=300, H=128, E=8, R=2, K=4, A=128, router="topk", seed=84)
    run_case(wl, I=384, N=256, col_major=True)


@pytest.mark.parametrize("col_major", [False, True])
def test_chain_from_fp8_dispatch(col_major):
    """The FP8 dispatch's own codes and scales feed the GEMM (inner = hidden)."""
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=512, H=512, E=8, R=2, K=4, A=128, router="topk", seed=85)
    g = gpu_layout(wl)
    try:
        if col_major:
            ep.ep_set_scale_layout(g.handle, ep.EP_SCALES_COL_MAJOR_TMA)
        cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A)
        q = torch.empty((g.cap, wl.H), dtype=torch.uint8, device=dev)
        s = torch.empty(ep.ep_scale_buffer_floats(cfg, ep.EP_SCALES_COL_MAJOR_TMA if col_major
                                                  else ep.EP_SCALES_ROW_MAJOR), dtype=torch.float32, device=dev)
        ep.ep_dispatch_fp8(g.handle, wl.x.to(dev), q, s)
        rng = np.random.default_rng(86)
        N = 512
        wq, ws = expert_weights(rng, wl.E, N, wl.H)
        out = run_gemm(g, wl, q, s, wl.H, wq, ws, N)
        o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A)
        oq, osc = oracle.dispatch_fp8(workloads.bf16_bits(wl.x), o.row_src[:o.rows])
        ref = oracle.expert_combine_fp8(oq, osc, wq, ws, wl.topk_idx.numpy(), o.pos, wl.topk_weights.numpy())
        combine_close(out, ref)
    finally:
        ep.ep_handle_destroy(g.handle)


def test_bench_shape():
    """The shape the bench times: 32 local experts, 4096 tokens x top-8,
    alignment 128, inner 2048 -> 7168 outputs: 16 k-blocks per tile over 28
    column blocks and ~288 row tiles.  96 tokens (both ends and a seeded
    sample), all 7168 columns each."""
    wl = workloads.generate(None, T=4096, H=7168, E=32, R=8, K=8, A=128, router="topk", seed=5, with_x=False)
    rng = np.random.default_rng(18)
    tok = np.unique(np.concatenate([np.arange(16), np.arange(4080, 4096), rng.integers(16, 4080, 64)]))
    run_case(wl, I=2048, N=7168, check_tokens=tok, seed=6)


def test_rejects_bad_shapes():
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=64, H=128, E=8, R=2, K=2, A=128, router="topk", seed=87)
    g = gpu_layout(wl)
    try:
        aq = torch.zeros((g.cap, 192), dtype=torch.uint8, device=dev)
        sa = torch.ones((g.cap, 2), dtype=torch.float32, device=dev)
        wq = torch.zeros((8, 256, 192), dtype=torch.uint8, device=dev)
        ws = torch.ones((8, 2, 2), dtype=torch.float32, device=dev)
        acc = torch.zeros((64, 256), dtype=torch.float32, device=dev)
        out = torch.zeros((64, 256), dtype=torch.bfloat16, device=dev)
        tw = wl.topk_weights.to(dev)
        for args in [(aq, sa, 192, wq, ws, 256), (aq, None, 128, wq, ws, 256), (aq, sa, 128, wq, None, 256),
                     (aq, sa, 128, wq, ws, 128)]:
            with pytest.raises(ep.EpError) as e:
                ep.ep_expert_combine_fp8(g.handle, *args, tw, acc, out)
            assert e.value.code == ep.EP_ERR_ARG
    finally:
        ep.ep_handle_destroy(g.handle)
