"""Parity of the low-latency (static, masked) path with the oracle.

ep_ll_dispatch / ep_ll_dispatch_fp8 / ep_ll_combine through the C ABI against
oracle.ll_layout + the oracle's dispatch and combine: pos, recv_count, the
used slots (bit-exact bf16, FP8 codes and scales) and combine within
rtol 1e-2 / atol 1e-3.  Slots past recv_count must stay untouched.
"""
import numpy as np
import pytest
import torch

import combine_ep_get_08_b200 as ep
import oracle
import workloads
from ep_harness import combine_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_ep_get_08_b200 import build_lib
    build_lib.build()
    oracle.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_ll(wl, M, fp8, idx=None, want_status=0, col_major=False):
    dev = torch.device("cuda")
    idx = wl.topk_idx if idx is None else idx
    idx_np = idx.numpy()
    o = oracle.ll_layout(idx_np, wl.E, M)
    cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, 1)
    h = ep.ep_ll_handle_create(cfg, M)
    try:
        cap = ep.ep_ll_capacity_rows(cfg, M)
        assert cap == wl.E * M
        if col_major:
            ep.ep_set_scale_layout(h, ep.EP_SCALES_COL_MAJOR_TMA)
        x_d, idx_d = wl.x.to(dev), idx.to(dev)
        cnt = torch.full((wl.E,), -9, dtype=torch.int32, device=dev)
        nb = wl.H // 128
        if fp8:
            q = torch.full((cap, wl.H), 0x5A, dtype=torch.uint8, device=dev)
            nsc = ep.ep_ll_scale_buffer_floats(cfg, M, ep.EP_SCALES_COL_MAJOR_TMA if col_major else 0)
            sc = torch.full((nsc,), -3.0, dtype=torch.float32, device=dev)
            ep.ep_ll_dispatch_fp8(h, idx_d, x_d, q, sc, cnt)
        else:
            recv = torch.full((cap, wl.H), 12345, dtype=torch.int16, device=dev).view(torch.bfloat16)
            ep.ep_ll_dispatch(h, idx_d, x_d, recv, cnt)
        pos = torch.full((wl.T, wl.K), -9, dtype=torch.int32, device=dev)
        ep.ep_copy_routing(h, pos)
        assert ep.ep_get_status(h) == want_status
        np.testing.assert_array_equal(pos.cpu().numpy(), o.pos, err_msg="pos")
        np.testing.assert_array_equal(cnt.cpu().numpy(), o.recv_count, err_msg="recv_count")
        used = np.flatnonzero(o.row_src >= 0).astype(np.int32)
        free = np.flatnonzero(o.row_src < 0)
        xb = workloads.bf16_bits(wl.x)
        used_d = torch.from_numpy(used).long().to(dev)
        free_d = torch.from_numpy(free).long().to(dev)
        if fp8:
            oq, osc = oracle.dispatch_fp8(xb, o.row_src, used)
            np.testing.assert_array_equal(q[used_d].cpu().numpy(), oq, err_msg="fp8 codes")
            if col_major:
                ldm = (M + 3) // 4 * 4
                s3 = sc.view(wl.E, nb, ldm)
                got = s3[used_d // M, :, used_d % M]                   # [n, NB]
            else:
                got = sc.view(cap, nb)[used_d]
            np.testing.assert_array_equal(got.cpu().numpy().view(np.uint32), osc.view(np.uint32),
                                          err_msg="fp8 scales")
            if len(free):
                assert bool((q[free_d] == 0x5A).all()), "masked slots written"
        else:
            np.testing.assert_array_equal(workloads.bf16_bits(recv[used_d]),
                                          oracle.dispatch_bf16(xb, o.row_src, used), err_msg="bf16 rows")
            if len(free):
                assert bool((recv[free_d].view(torch.int16) == 12345).all()), "masked slots written"
        # combine of stand-in expert outputs in the slots
        gen = torch.Generator(device=dev)
        gen.manual_seed(5)
        y = torch.randn((cap, wl.H), generator=gen, device=dev).to(torch.bfloat16)
        w_d = wl.topk_weights.to(dev)
        out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
        ep.ep_ll_combine(h, y, w_d, out)
        if wl.T:
            ref = oracle.combine(workloads.bf16_bits(y), o.pos, wl.topk_weights.numpy())
            combine_close(out, ref)
        assert ep.ep_get_status(h) == want_status
    finally:
        ep.ep_handle_destroy(h)


CASES = [
    dict(T=128, H=7168, E=256, R=32, K=8, router="topk", seed=41, M=128),     # decode shape
    dict(T=128, H=7168, E=256, R=32, K=8, router="topk", seed=42, M=256),
    dict(T=37, H=200, E=32, R=4, K=4, router="uniform", seed=43, M=40),       # ragged row
    dict(T=1, H=128, E=8, R=2, K=2, router="topk", seed=44, M=1),
    dict(T=33, H=256, E=1024, R=128, K=64, router="topk", seed=45, M=33),     # max E, max K
    dict(T=256, H=2048, E=64, R=8, K=6, router="zipf", seed=46, M=256),       # skewed experts
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"T{c['T']}H{c['H']}E{c['E']}K{c['K']}M{c['M']}")
@pytest.mark.parametrize("fp8", [False, True])
def test_ll_parity(case, fp8):
    case = dict(case)
    M = case.pop("M")
    wl = workloads.generate(None, A=1, **case)
    if fp8 and wl.H % 128:
        pytest.skip("FP8 needs H % 128 == 0")
    run_ll(wl, M, fp8)


def test_ll_col_major_scales():
    wl = workloads.generate(None, T=100, H=1024, E=16, R=4, K=4, A=1, router="topk", seed=47)
    run_ll(wl, 101, True, col_major=True)


def test_ll_masked_and_invalid_ids():
    wl = workloads.generate(None, T=64, H=512, E=16, R=4, K=4, A=1, router="topk", seed=48)
    idx = wl.topk_idx.clone()
    idx[torch.rand(idx.shape, generator=torch.Generator().manual_seed(1)) < 0.3] = -1
    run_ll(wl, 64, False, idx=idx)
    run_ll(wl, 64, True, idx=idx)
    bad = wl.topk_idx.clone()
    bad[5, 2] = 16
    o = oracle.ll_layout(bad.numpy(), wl.E, 64)
    assert o.status == oracle.BAD_EXPERT
    dev = torch.device("cuda")
    cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, 1)
    h = ep.ep_ll_handle_create(cfg, 64)
    try:
        recv = torch.empty((wl.E * 64, wl.H), dtype=torch.bfloat16, device=dev)
        ep.ep_ll_dispatch(h, bad.to(dev), wl.x.to(dev), recv)
        assert ep.ep_get_status(h) & ep.EP_DEV_BAD_EXPERT
        pos = torch.empty((wl.T, wl.K), dtype=torch.int32, device=dev)
        ep.ep_copy_routing(h, pos)
        assert int(pos[5, 2]) == -1
    finally:
        ep.ep_handle_destroy(h)


def test_ll_slot_overflow():
    """Repeated experts in a token can exceed M: the pairs past the M-th drop."""
    wl = workloads.generate(None, T=10, H=256, E=8, R=2, K=4, A=1, router="topk", seed=49)
    idx = torch.full((10, 4), 3, dtype=torch.int64)
    idx[:, 1] = torch.arange(10) % 8
    o = oracle.ll_layout(idx.numpy(), wl.E, 12)
    assert o.status == oracle.SLOT_OVERFLOW
    run_ll(wl, 12, False, idx=idx, want_status=ep.EP_DEV_SLOT_OVERFLOW)


def test_ll_empty_batch():
    dev = torch.device("cuda")
    cfg = ep.make_config(0, 256, 8, 2, 2, 1)
    h = ep.ep_ll_handle_create(cfg, 4)
    try:
        cnt = torch.full((8,), 7, dtype=torch.int32, device=dev)
        recv = torch.empty((32, 256), dtype=torch.bfloat16, device=dev)
        ep.ep_ll_dispatch(h, None, None, recv, cnt)
        assert not cnt.any()
        ep.ep_ll_combine(h, recv, None, None)
        assert ep.ep_get_status(h) == 0
    finally:
        ep.ep_handle_destroy(h)


def test_ll_mode_checks():
    cfg = ep.make_config(16, 256, 8, 2, 2, 1)
    with pytest.raises(ep.EpError):
        ep.ep_ll_handle_create(cfg, 8)                 # T > M
    h = ep.ep_ll_handle_create(cfg, 16)
    hn = ep.ep_handle_create(cfg)
    dev = torch.device("cuda")
    try:
        idx = torch.zeros((16, 2), dtype=torch.int64, device=dev)
        with pytest.raises(ep.EpError) as e:
            ep.ep_get_layout(h, idx)
        assert e.value.code == ep.EP_ERR_STATE
        recv = torch.empty((8 * 16, 256), dtype=torch.bfloat16, device=dev)
        x = torch.zeros((16, 256), dtype=torch.bfloat16, device=dev)
        with pytest.raises(ep.EpError) as e:
            ep.ep_ll_dispatch(hn, idx, x, recv)
        assert e.value.code == ep.EP_ERR_STATE
        with pytest.raises(ep.EpError) as e:
            ep.ep_ll_combine(h, recv, torch.zeros((16, 2), device=dev), x)   # before any dispatch
        assert e.value.code == ep.EP_ERR_STATE
    finally:
        ep.ep_handle_destroy(h)
        ep.ep_handle_destroy(hn)


def test_ll_cuda_graph_replay():
    """Static buffers: one captured dispatch + combine serves new routings."""
    dev = torch.device("cuda")
    T, H, E, K, M = 64, 1024, 32, 4, 64
    wls = [workloads.generate(None, T=T, H=H, E=E, R=4, K=K, A=1, router="topk", seed=60 + i)
           for i in range(3)]
    cfg = ep.make_config(T, H, E, 4, K, 1)
    h = ep.ep_ll_handle_create(cfg, M)
    try:
        idx_d = wls[0].topk_idx.to(dev)
        x_d = wls[0].x.to(dev)
        w_d = wls[0].topk_weights.to(dev)
        recv = torch.zeros((E * M, H), dtype=torch.bfloat16, device=dev)
        cnt = torch.zeros((E,), dtype=torch.int32, device=dev)
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):                       # warm up outside the capture
            ep.ep_ll_dispatch(h, idx_d, x_d, recv, cnt)
            ep.ep_ll_combine(h, recv, w_d, out)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            ep.ep_ll_dispatch(h, idx_d, x_d, recv, cnt)
            ep.ep_ll_combine(h, recv, w_d, out)
        for wl in wls[1:] + wls[:1]:
            idx_d.copy_(wl.topk_idx)
            x_d.copy_(wl.x)
            w_d.copy_(wl.topk_weights)
            g.replay()
            torch.cuda.synchronize()
            o = oracle.ll_layout(wl.topk_idx.numpy(), E, M)
            np.testing.assert_array_equal(cnt.cpu().numpy(), o.recv_count)
            recv_bits = workloads.bf16_bits(recv)
            ref = oracle.combine(recv_bits, o.pos, wl.topk_weights.numpy())
            combine_close(out, ref)
            # identity experts: out = x * sum of weights
            x64 = (workloads.bf16_bits(wl.x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            combine_close(out, x64 * wl.topk_weights.numpy().astype(np.float64).sum(1, keepdims=True))
        del g
        assert ep.ep_get_status(h) == 0
    finally:
        ep.ep_handle_destroy(h)
