"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: layout (counts, membership, offsets, pos, row_src/row_slot,
row_weight), bf16 received rows, FP8 codes and scales.  Combine within
rtol 1e-2 / atol 1e-3 of the oracle's fp64 weighted sum.
"""
import numpy as np
import pytest
import torch

import combine_ep_get_08_b200 as ep
import oracle
import workloads
from ep_harness import ROW_CHUNK, TOKEN_CHUNK, assert_layout_equal, chunks as _chunks, combine_close, config_of, gpu_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_ep_get_08_b200 import build_lib
    build_lib.build()
    oracle.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_full(wl, fp8: bool, y_seed=99, check_rows=None, check_tokens=None, sm_limit=0):
    """Layout + dispatch + combine on the GPU, compared with the oracle.

    check_rows / check_tokens: compare only these received rows / tokens
    (indexing happens on the device); None compares every row and every
    token, in chunks so that host memory stays bounded at any size.
    sm_limit: cap on the SMs dispatch and combine occupy (0: all)."""
    dev = torch.device("cuda")
    idx, w = wl.topk_idx.numpy(), wl.topk_weights.numpy()
    o = oracle.layout(idx, wl.E, wl.R, wl.A, topk_weights=w)
    assert o.status == 0
    g = gpu_layout(wl)
    try:
        assert_layout_equal(g, o)
        if sm_limit:
            ep.ep_set_sm_limit(g.handle, sm_limit)
        x_d = wl.x.to(dev)
        xb = workloads.bf16_bits(wl.x)
        cap = g.cap
        sel = np.arange(g.rows, dtype=np.int32) if check_rows is None else np.asarray(check_rows, np.int32)
        if fp8:
            q = torch.full((max(cap, 1), wl.H), 0x5A, dtype=torch.uint8, device=dev)
            s = torch.full((max(cap, 1), wl.H // 128), -3.0, dtype=torch.float32, device=dev)
            ep.ep_dispatch_fp8(g.handle, x_d, q, s)
            for part in _chunks(sel, ROW_CHUNK):
                part_d = torch.from_numpy(part).long().to(dev)
                oq, osc = oracle.dispatch_fp8(xb, o.row_src, part)
                np.testing.assert_array_equal(q[part_d].cpu().numpy(), oq, err_msg="fp8 codes")
                np.testing.assert_array_equal(s[part_d].cpu().numpy().view(np.uint32), osc.view(np.uint32),
                                              err_msg="fp8 scales")
            if cap > g.rows:                      # rows beyond `rows` are untouched
                assert bool((q[g.rows:cap] == 0x5A).all())
                assert bool((s[g.rows:cap] == -3.0).all())
            del q, s
        else:
            recv = torch.full((max(cap, 1), wl.H), 12345, dtype=torch.int16, device=dev).view(torch.bfloat16)
            ep.ep_dispatch(g.handle, x_d, recv)
            for part in _chunks(sel, ROW_CHUNK):
                part_d = torch.from_numpy(part).long().to(dev)
                np.testing.assert_array_equal(workloads.bf16_bits(recv[part_d]),
                                              oracle.dispatch_bf16(xb, o.row_src, part), err_msg="bf16 rows")
            if cap > g.rows:
                assert bool((recv[g.rows:cap].view(torch.int16) == 12345).all())
            del recv
        # combine of stand-in expert outputs y [cap, H] (seeded N(0,1), made on the device)
        gen = torch.Generator(device=dev)
        gen.manual_seed(y_seed)
        y_d = torch.randn((max(cap, 1), wl.H), generator=gen, device=dev).to(torch.bfloat16)
        w_d = wl.topk_weights.to(dev)
        out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
        ep.ep_combine(g.handle, y_d, w_d, out)
        tsel = np.arange(wl.T, dtype=np.int32) if check_tokens is None else np.asarray(check_tokens, np.int32)
        for part in _chunks(tsel, TOKEN_CHUNK):
            need = o.pos[part]                     # [n, K] rows those tokens read (-1: masked slot)
            uniq, inv = np.unique(need[need >= 0], return_inverse=True)
            small_pos = np.full(need.shape, -1, np.int32)
            small_pos[need >= 0] = inv
            y_small = workloads.bf16_bits(y_d[torch.from_numpy(uniq).long().to(dev)]) if len(uniq) \
                else np.zeros((1, wl.H), np.uint16)
            ref = oracle.combine(y_small, small_pos, w[part])
            combine_close(out[torch.from_numpy(part).long().to(dev)], ref)
        assert ep.ep_get_status(g.handle) == 0
    finally:
        ep.ep_handle_destroy(g.handle)


SMALL = [
    dict(name="tiny"),
    dict(T=1000, H=7168, E=64, R=4, K=6, A=3, router="topk", seed=21),
    dict(T=777, H=200, E=32, R=8, K=4, A=1, router="uniform", seed=22),      # ragged row (25 vectors)
    dict(T=513, H=384, E=256, R=32, K=8, A=16, router="group", seed=23),
    dict(T=33, H=128, E=1024, R=128, K=64, A=2, router="topk", seed=24),      # max E, max K, R > 64
    dict(T=1, H=8, E=1, R=1, K=1, A=1, router="topk", seed=25),
    dict(T=300, H=1024, E=8, R=2, K=8, A=300, router="topk", seed=26),      # A > T*K/E
    dict(T=20000, H=64, E=64, R=8, K=8, A=4, router="topk", seed=27),        # beyond one cluster: cooperative
    dict(T=16384, H=64, E=256, R=64, K=8, A=2, router="group", seed=28),     # 131072 pairs: cooperative
    dict(T=8192, H=64, E=256, R=64, K=8, A=2, router="group", seed=30),      # 16-CTA cluster, 4096 pairs each
    # K = 64: a token's destinations fill a whole stage slot (256 bytes)
    dict(T=12000, H=128, E=128, R=8, K=64, A=1, router="topk", seed=29),
    # K % 4 != 0 on the chunked dispatch: destination spans start inside a
    # 16-byte word (1 200 tokens fill the GPU: chunked, not the register kernel)
    dict(T=1200, H=512, E=64, R=8, K=6, A=5, router="topk", seed=32),
    dict(T=1201, H=256, E=32, R=4, K=3, A=2, router="uniform", seed=33),
]


def _wl(spec):
    spec = dict(spec)
    name = spec.pop("name", None)
    return workloads.generate(name, **spec)


@pytest.mark.parametrize("spec", SMALL, ids=lambda s: s.get("name") or f"T{s['T']}H{s['H']}E{s['E']}K{s['K']}A{s['A']}")
@pytest.mark.parametrize("fp8", [False, True])
def test_small_parity(spec, fp8):
    wl = _wl(spec)
    if fp8 and wl.H % 128:
        pytest.skip("FP8 needs H % 128 == 0")
    run_full(wl, fp8)


@pytest.mark.parametrize("name", ["dsv3", "decode", "skew", "large"])
def test_full_size_parity(name):
    """Full-size workloads, same seeds and launch configuration as the bench:
    every layout array, every received row (bf16 rows, or FP8 codes and
    scales) and every combined token against the oracle."""
    wl = workloads.generate(name)
    run_full(wl, wl.fp8)
    if name == "dsv3":
        # the bench's dsv3 step is bf16; the FP8 dispatch on the same routing too
        run_full(wl, True)


def test_identity_round_trip_bf16():
    """combine(dispatch(x)) with identity experts returns x * sum_k w."""
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=2048, H=7168, E=256, R=8, K=8, A=1, router="group", seed=31)
    g = gpu_layout(wl)
    try:
        x_d = wl.x.to(dev)
        recv = torch.empty((g.cap, wl.H), dtype=torch.bfloat16, device=dev)
        ep.ep_dispatch(g.handle, x_d, recv)
        out = torch.empty_like(x_d)
        ep.ep_combine(g.handle, recv, wl.topk_weights.to(dev), out)
        ref = wl.x.double().numpy() * wl.topk_weights.double().numpy().sum(1, keepdims=True)
        combine_close(out, ref)
    finally:
        ep.ep_handle_destroy(g.handle)


def test_handle_reuse_and_determinism():
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=600, H=1024, E=64, R=8, K=8, A=4, router="topk", seed=41)
    g = gpu_layout(wl)
    try:
        g2 = gpu_layout(wl, handle=g.handle)      # same handle, second layout: identical bytes
        for key in ("pos", "row_src", "row_slot", "expert_offsets"):
            np.testing.assert_array_equal(getattr(g, key), getattr(g2, key))
        o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A)
        for seed in (1, 2, 3):                     # three dispatches on one layout
            x = workloads.bf16_normal(np.random.default_rng(seed), wl.T, wl.H)
            recv = torch.empty((g.cap, wl.H), dtype=torch.bfloat16, device=dev)
            ep.ep_dispatch(g.handle, x.to(dev), recv)
            np.testing.assert_array_equal(workloads.bf16_bits(recv[:g.rows]),
                                          oracle.dispatch_bf16(workloads.bf16_bits(x), o.row_src))
    finally:
        ep.ep_handle_destroy(g.handle)


def test_empty_batch():
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=0, H=256, E=16, R=4, K=2, A=8, router="topk", seed=1)
    g = gpu_layout(wl)
    try:
        assert g.rows == 0 and g.status == 0
        assert (g.expert_offsets == 0).all() and (g.num_tokens_per_expert == 0).all()
        x = torch.empty((0, wl.H), dtype=torch.bfloat16, device=dev)
        ep.ep_dispatch(g.handle, x, x)
        ep.ep_combine(g.handle, x, torch.empty((0, 2), device=dev), x)
    finally:
        ep.ep_handle_destroy(g.handle)


def test_repeated_experts_in_a_row():
    wl = workloads.generate(None, T=100, H=256, E=8, R=2, K=4, A=2, router="topk", seed=3)
    idx = wl.topk_idx.clone()
    idx[:, 1] = idx[:, 0]                         # every token names its first expert twice
    wl.topk_idx = idx
    run_full(wl, False)
    run_full(wl, True)


def test_invalid_expert_id_sets_status():
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=50, H=256, E=16, R=4, K=2, A=1, router="uniform", seed=4)
    idx = wl.topk_idx.clone()
    idx[7, 1] = 16
    idx[9, 0] = -1
    g = gpu_layout(wl, idx_d=idx.to(dev))
    try:
        assert g.status & ep.EP_DEV_BAD_EXPERT
        assert g.pos[7, 1] == -1 and g.pos[9, 0] == -1
        assert int(g.num_tokens_per_expert.sum()) == 50 * 2 - 2
        # dispatch/combine skip the invalid pairs and stay in bounds
        x_d = wl.x.to(dev)
        recv = torch.zeros((g.cap, wl.H), dtype=torch.bfloat16, device=dev)
        ep.ep_dispatch(g.handle, x_d, recv)
        out = torch.empty_like(x_d)
        ep.ep_combine(g.handle, recv, wl.topk_weights.to(dev), out)
        torch.cuda.synchronize()
        ep.ep_clear_status(g.handle)
        assert ep.ep_get_status(g.handle) == 0
    finally:
        ep.ep_handle_destroy(g.handle)


def test_bounded_wait_gives_up():
    """A grid-wide wait that can never complete ends after its limit with
    EP_DEV_WAIT_TIMEOUT; after ep_clear_status the handle works again.
    160 000 pairs exceed one cluster (16 CTAs x 8192 pairs), so the layout
    takes the cooperative kernel, the one with a grid-wide wait."""
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=20000, H=64, E=64, R=8, K=8, A=1, router="topk", seed=5)
    cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A)
    h = ep.ep_handle_create(cfg)
    try:
        ep.ep_set_wait_limit(h, 20_000_000, 1)     # 20 ms, one CTA that never arrives
        idx_d = wl.topk_idx.to(dev)
        ep.ep_get_layout(h, idx_d)
        assert ep.ep_get_status(h) & ep.EP_DEV_WAIT_TIMEOUT
        ep.ep_set_wait_limit(h, 1_000_000_000, 0)
        ep.ep_clear_status(h)
        g = gpu_layout(wl, handle=h, with_weights=False)
        assert g.status == 0
        o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A)
        assert_layout_equal(g, o, with_weights=False)
    finally:
        ep.ep_handle_destroy(h)


def test_host_argument_errors():
    dev = torch.device("cuda")
    cfg = ep.make_config(16, 256, 8, 2, 2, 1)
    h = ep.ep_handle_create(cfg)
    try:
        x = torch.zeros((16, 256), dtype=torch.bfloat16, device=dev)
        with pytest.raises(ep.EpError) as ei:
            ep.ep_dispatch(h, x, x)               # no layout yet
        assert ei.value.code == ep.EP_ERR_STATE
        idx = torch.zeros((16, 2), dtype=torch.int64, device=dev)
        ep.ep_get_layout(h, idx)
        recv = torch.zeros((40, 256), dtype=torch.bfloat16, device=dev)
        with pytest.raises(ep.EpError) as ei:
            ep.ep_dispatch(h, x.data_ptr() + 2, recv)   # misaligned
        assert ei.value.code == ep.EP_ERR_ARG
        with pytest.raises(ep.EpError) as ei:
            ep.ep_dispatch_fp8(h, x, recv, None)  # FP8 without a scale buffer
        assert ei.value.code == ep.EP_ERR_ARG
    finally:
        ep.ep_handle_destroy(h)
    with pytest.raises(ep.EpError):
        ep.ep_handle_create(ep.make_config(16, 256, 9, 2, 2, 1))   # E % R != 0


@pytest.mark.parametrize("sms", [1, 7, 24])
@pytest.mark.parametrize("fp8", [False, True])
def test_sm_limit_parity(sms, fp8):
    """Dispatch and combine capped to a few SMs (ep_set_sm_limit, the num_sms
    budget of bowenzhou.top "deepep/01-overview" section 1.1) against the
    oracle.  With one SM the chunked dispatch runs in one CTA, which claims
    every row part of the 1200 tokens in turn and wraps its 16-stage ring
    ~150 times; the combine grid shrinks to the cap."""
    wl = workloads.generate(None, T=1200, H=2048, E=64, R=8, K=8, A=4, router="topk", seed=61)
    run_full(wl, fp8, sm_limit=sms)


def test_masked_slots_parity():
    """-1 slots (tokens that select fewer than K experts): no row, nothing in combine."""
    wl = workloads.generate(None, T=900, H=1024, E=64, R=8, K=8, A=4, router="topk", seed=71)
    idx = wl.topk_idx.clone()
    g = torch.Generator().manual_seed(5)
    idx[torch.rand(idx.shape, generator=g) < 0.25] = -1
    idx[3, :] = -1                                 # one token with no expert at all
    wl.topk_idx = idx
    run_full(wl, False)
    run_full(wl, True)


def test_col_major_tma_scales():
    """The column-major, 4-float-aligned scale layout holds the same values."""
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=333, H=1024, E=32, R=4, K=6, A=8, router="topk", seed=81)
    g = gpu_layout(wl)
    try:
        cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A)
        nb = wl.H // 128
        ld = (g.cap + 3) // 4 * 4
        assert ep.ep_scale_buffer_floats(cfg, ep.EP_SCALES_COL_MAJOR_TMA) == nb * ld
        x = wl.x.to(dev)
        q_r = torch.zeros((g.cap, wl.H), dtype=torch.uint8, device=dev)
        s_r = torch.zeros((g.cap, nb), dtype=torch.float32, device=dev)
        ep.ep_dispatch_fp8(g.handle, x, q_r, s_r)
        ep.ep_set_scale_layout(g.handle, ep.EP_SCALES_COL_MAJOR_TMA)
        q_c = torch.zeros((g.cap, wl.H), dtype=torch.uint8, device=dev)
        s_c = torch.full((nb, ld), -1.0, dtype=torch.float32, device=dev)
        ep.ep_dispatch_fp8(g.handle, x, q_c, s_c)
        torch.cuda.synchronize()
        assert torch.equal(q_r[:g.rows], q_c[:g.rows])
        assert torch.equal(s_r[:g.rows].t().contiguous().view(torch.int32), s_c[:, :g.rows].contiguous().view(torch.int32))
        assert (s_c.data_ptr() % 16 == 0) and (ld * 4) % 16 == 0     # every block column 16-byte aligned
        o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A)
        oq, osc = oracle.dispatch_fp8(workloads.bf16_bits(wl.x), o.row_src)
        np.testing.assert_array_equal(s_c[:, :g.rows].t().cpu().numpy().view(np.uint32), osc.view(np.uint32))
    finally:
        ep.ep_handle_destroy(g.handle)


@pytest.mark.parametrize("T", [1, 13, 64, 295])
def test_small_batch_layout(T):
    """ep_get_layout of a batch with fewer than two tokens per SM runs the
    small-batch kernel without its copy (one CTA per token, each counting all
    pairs); under a 5-SM cap (T = 13) five CTAs handle 2-3 tokens each."""
    wl = workloads.generate(None, T=T, H=256, E=64, R=8, K=8, A=4, router="topk", seed=300 + T)
    h = ep.ep_handle_create(config_of(wl))
    if T == 13:
        ep.ep_set_sm_limit(h, 5)
    g = gpu_layout(wl, handle=h)
    try:
        assert g.status == 0
        o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A, topk_weights=wl.topk_weights.numpy())
        assert_layout_equal(g, o)
    finally:
        ep.ep_handle_destroy(h)

