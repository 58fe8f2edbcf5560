"""Parity of the fused layout + dispatch (ep_layout_dispatch, _fp8) with the oracle.

One call computes the layout (counts pre-pass; per-chunk ranks and decoupled
look-back inside the dispatch) and the dispatch.  Checked bit-exactly against
the CPU oracle: every layout array (the caller's copies and the handle's
routing arrays), every received row (bf16 rows, or FP8 codes and scales),
untouched rows past `rows`; then ep_combine on the same handle against the
oracle within rtol 1e-2 / atol 1e-3 (the handle the fused call filled serves
the combine, and further plain dispatches).
"""
import numpy as np
import pytest
import torch

import combine_ep_get_08_b200 as ep
import oracle
import workloads
from ep_harness import ROW_CHUNK, TOKEN_CHUNK, chunks as _chunks, combine_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_ep_get_08_b200 import build_lib
    build_lib.build()
    oracle.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def fused(h, wl, fp8, idx_d=None, w_d=None, x_d=None, with_weights=True):
    """One fused call on h; returns (layout outputs, received buffers) on the device."""
    dev = torch.device("cuda")
    cap = ep.ep_capacity_rows(ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A))
    idx_d = wl.topk_idx.to(dev) if idx_d is None else idx_d
    w_d = (wl.topk_weights.to(dev) if with_weights else None) if w_d is None else w_d
    x_d = wl.x.to(dev) if x_d is None else x_d
    outs = dict(num_tokens_per_expert=torch.full((wl.E,), -9, dtype=torch.int32, device=dev),
                num_tokens_per_rank=torch.full((wl.R,), -9, dtype=torch.int32, device=dev),
                is_token_in_rank=torch.full((wl.T, wl.R), 7, dtype=torch.uint8, device=dev),
                expert_offsets=torch.full((wl.E + 1,), -9, dtype=torch.int32, device=dev),
                rank_offsets=torch.full((wl.R + 1,), -9, dtype=torch.int32, device=dev))
    if fp8:
        q = torch.full((max(cap, 1), wl.H), 0x5A, dtype=torch.uint8, device=dev)
        s = torch.full((max(cap, 1), wl.H // 128), -3.0, dtype=torch.float32, device=dev)
        ep.ep_layout_dispatch_fp8(h, idx_d, w_d, x_d, q, s, **outs)
        recv = (q, s)
    else:
        r = torch.full((max(cap, 1), wl.H), 12345, dtype=torch.int16, device=dev).view(torch.bfloat16)
        ep.ep_layout_dispatch(h, idx_d, w_d, x_d, r, **outs)
        recv = (r,)
    return outs, recv, cap


def check_layout(h, wl, outs, o, with_weights=True):
    dev = torch.device("cuda")
    cap = o.capacity
    pos = torch.full((wl.T, wl.K), -9, dtype=torch.int32, device=dev)
    src = torch.full((max(cap, 1),), -9, dtype=torch.int32, device=dev)
    slot = torch.full((max(cap, 1),), -9, dtype=torch.int32, device=dev)
    wt = torch.full((max(cap, 1),), -9.0, dtype=torch.float32, device=dev)
    ep.ep_copy_routing(h, pos, src, slot, wt)
    rows = ep.ep_get_num_rows(h)
    assert rows == o.rows
    for k in ("num_tokens_per_expert", "num_tokens_per_rank", "is_token_in_rank", "expert_offsets", "rank_offsets"):
        np.testing.assert_array_equal(outs[k].cpu().numpy(), getattr(o, k).reshape(outs[k].shape), err_msg=k)
    np.testing.assert_array_equal(pos.cpu().numpy(), o.pos, err_msg="pos")
    np.testing.assert_array_equal(src[:rows].cpu().numpy(), o.row_src, err_msg="row_src")
    np.testing.assert_array_equal(slot[:rows].cpu().numpy(), o.row_slot, err_msg="row_slot")
    if with_weights:
        np.testing.assert_array_equal(wt[:rows].cpu().numpy().view(np.uint32), o.row_weight.view(np.uint32),
                                      err_msg="row_weight")
    return rows


def check_rows(wl, recv, o, fp8, cap):
    dev = torch.device("cuda")
    xb = workloads.bf16_bits(wl.x)
    rows = o.rows
    for part in _chunks(np.arange(rows, dtype=np.int32), ROW_CHUNK):
        part_d = torch.from_numpy(part).long().to(dev)
        if fp8:
            oq, osc = oracle.dispatch_fp8(xb, o.row_src, part)
            np.testing.assert_array_equal(recv[0][part_d].cpu().numpy(), oq, err_msg="fp8 codes")
            np.testing.assert_array_equal(recv[1][part_d].cpu().numpy().view(np.uint32), osc.view(np.uint32),
                                          err_msg="fp8 scales")
        else:
            np.testing.assert_array_equal(workloads.bf16_bits(recv[0][part_d]),
                                          oracle.dispatch_bf16(xb, o.row_src, part), err_msg="bf16 rows")
    if cap > rows:
        if fp8:
            assert bool((recv[0][rows:cap] == 0x5A).all()) and bool((recv[1][rows:cap] == -3.0).all())
        else:
            assert bool((recv[0][rows:cap].view(torch.int16) == 12345).all())


def check_combine(h, wl, o, cap, seed=99):
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    y_d = torch.randn((max(cap, 1), wl.H), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
    ep.ep_combine(h, y_d, wl.topk_weights.to(dev), out)
    w = wl.topk_weights.numpy()
    for part in _chunks(np.arange(wl.T, dtype=np.int32), TOKEN_CHUNK):
        need = o.pos[part]
        uniq, inv = np.unique(need[need >= 0], return_inverse=True)
        small_pos = np.full(need.shape, -1, np.int32)
        small_pos[need >= 0] = inv
        y_small = workloads.bf16_bits(y_d[torch.from_numpy(uniq).long().to(dev)]) if len(uniq) \
            else np.zeros((1, wl.H), np.uint16)
        combine_close(out[torch.from_numpy(part).long().to(dev)], oracle.combine(y_small, small_pos, w[part]))


def run_fused(wl, fp8, sm_limit=0):
    idx, w = wl.topk_idx.numpy(), wl.topk_weights.numpy()
    o = oracle.layout(idx, wl.E, wl.R, wl.A, topk_weights=w)
    assert o.status == 0
    h = ep.ep_handle_create(ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A))
    try:
        if sm_limit:
            ep.ep_set_sm_limit(h, sm_limit)
        outs, recv, cap = fused(h, wl, fp8)
        assert ep.ep_get_status(h) == 0
        check_layout(h, wl, outs, o)
        check_rows(wl, recv, o, fp8, cap)
        del recv
        check_combine(h, wl, o, cap)
        assert ep.ep_get_status(h) == 0
    finally:
        ep.ep_handle_destroy(h)


CASES = [
    dict(name="tiny"),
    dict(T=1000, H=7168, E=64, R=4, K=6, A=3, router="topk", seed=21),
    dict(T=777, H=200, E=32, R=8, K=4, A=1, router="uniform", seed=22),       # ragged row (25 vectors)
    dict(T=513, H=384, E=256, R=32, K=8, A=16, router="group", seed=23),
    dict(T=33, H=128, E=1024, R=128, K=64, A=2, router="topk", seed=24),       # max E, max K, R > 64
    dict(T=1, H=8, E=1, R=1, K=1, A=1, router="topk", seed=25),
    dict(T=300, H=1024, E=8, R=2, K=8, A=300, router="topk", seed=26),       # A > T*K/E
    dict(T=20000, H=64, E=64, R=8, K=8, A=4, router="topk", seed=27),         # 148 chunks, 10 super-chunks
    dict(T=3000, H=128, E=128, R=8, K=64, A=1, router="topk", seed=29),       # 4096-pair chunks
    dict(T=400, H=128, E=1024, R=128, K=64, A=2, router="topk", seed=34),     # max E and K in the fused kernel
    dict(T=100, H=512, E=64, R=8, K=8, A=16, router="zipf", seed=35),        # small batch, padding rows
    dict(T=295, H=7168, E=256, R=32, K=8, A=1, router="topk", seed=36),       # largest small batch on 148 SMs
]
# Batches of fewer than two tokens per SM (tiny, T = 1, 33, 100, 295 above)
# take the single-launch small-batch kernel; the same checks apply.


@pytest.mark.parametrize("spec", CASES, ids=lambda s: s.get("name") or f"T{s['T']}H{s['H']}E{s['E']}K{s['K']}A{s['A']}")
@pytest.mark.parametrize("fp8", [False, True])
def test_fused_parity(spec, fp8):
    spec = dict(spec)
    name = spec.pop("name", None)
    wl = workloads.generate(name, **spec)
    if fp8 and wl.H % 128:
        pytest.skip("FP8 needs H % 128 == 0")
    run_fused(wl, fp8)


@pytest.mark.parametrize("name", ["dsv3", "decode", "skew", "large"])
def test_fused_full_size(name):
    """The bench workloads, every row and token compared."""
    wl = workloads.generate(name)
    run_fused(wl, wl.fp8)
    if name == "dsv3":
        run_fused(wl, True)


@pytest.mark.parametrize("sms", [1, 7])
@pytest.mark.parametrize("fp8", [False, True])
def test_fused_sm_limit(sms, fp8):
    """Fewer CTAs than chunks: each CTA takes several tickets in turn, so
    ring stages and phases carry over from one chunk to the next."""
    wl = workloads.generate(None, T=1200, H=2048, E=64, R=8, K=8, A=4, router="topk", seed=61)
    run_fused(wl, fp8, sm_limit=sms)


@pytest.mark.parametrize("fp8", [False, True])
def test_fused_kernel_small_batch(fp8):
    """A 64-token batch under a one-SM cap takes the fused kernel (two tokens
    per SM are enough): 64 one-token chunks, four super-chunks, one CTA."""
    wl = workloads.generate("tiny")
    run_fused(wl, fp8, sm_limit=1)


def test_fused_masked_and_repeated():
    wl = workloads.generate(None, T=900, H=1024, E=64, R=8, K=8, A=4, router="topk", seed=71)
    idx = wl.topk_idx.clone()
    g = torch.Generator().manual_seed(5)
    idx[torch.rand(idx.shape, generator=g) < 0.25] = -1
    idx[3, :] = -1                                 # a token with no expert at all
    idx[10:20, 1] = idx[10:20, 0]                  # repeated experts
    wl.topk_idx = idx
    run_fused(wl, False)
    run_fused(wl, True)


@pytest.mark.parametrize("fp8", [False, True])
def test_small_batch_masked_and_repeated(fp8):
    """The single-launch small-batch kernel with -1 slots, a token with no
    expert and repeated experts inside tokens."""
    wl = workloads.generate(None, T=120, H=1024, E=64, R=8, K=8, A=4, router="topk", seed=72)
    idx = wl.topk_idx.clone()
    g = torch.Generator().manual_seed(6)
    idx[torch.rand(idx.shape, generator=g) < 0.25] = -1
    idx[3, :] = -1
    idx[10:20, 1] = idx[10:20, 0]
    wl.topk_idx = idx
    run_fused(wl, fp8)


@pytest.mark.parametrize("fp8", [False, True])
def test_small_batch_fewer_ctas_than_tokens(fp8):
    """Under a 7-SM cap a 13-token batch still takes the small-batch kernel
    (fewer than two tokens per SM) with 7 CTAs: six of them handle two tokens
    each and carry their counts of earlier pairs from one token to the next."""
    wl = workloads.generate(None, T=13, H=512, E=16, R=4, K=4, A=4, router="topk", seed=74)
    run_fused(wl, fp8, sm_limit=7)


def test_small_batch_column_major_scales():
    """Column-major (TMA-aligned) scales from the small-batch kernel."""
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=90, H=1024, E=32, R=4, K=4, A=8, router="topk", seed=73)
    idx, w = wl.topk_idx.numpy(), wl.topk_weights.numpy()
    o = oracle.layout(idx, wl.E, wl.R, wl.A, topk_weights=w)
    cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A)
    h = ep.ep_handle_create(cfg)
    try:
        ep.ep_set_scale_layout(h, ep.EP_SCALES_COL_MAJOR_TMA)
        cap = ep.ep_capacity_rows(cfg)
        ld = (cap + 3) // 4 * 4
        q = torch.full((cap, wl.H), 0x5A, dtype=torch.uint8, device=dev)
        s = torch.full((ep.ep_scale_buffer_floats(cfg, ep.EP_SCALES_COL_MAJOR_TMA),), -3.0, dtype=torch.float32,
                       device=dev)
        ep.ep_layout_dispatch_fp8(h, wl.topk_idx.to(dev), wl.topk_weights.to(dev), wl.x.to(dev), q, s)
        assert ep.ep_get_status(h) == 0
        oq, osc = oracle.dispatch_fp8(workloads.bf16_bits(wl.x), o.row_src)
        np.testing.assert_array_equal(q[:o.rows].cpu().numpy(), oq)
        got = s.cpu().numpy().reshape(wl.H // 128, ld)[:, :o.rows].T
        np.testing.assert_array_equal(got.view(np.uint32), osc.view(np.uint32))
    finally:
        ep.ep_handle_destroy(h)


def test_small_batch_invalid_id_sets_status():
    """An id outside [0, E) other than -1 sets EP_DEV_BAD_EXPERT in the
    small-batch kernel too, and its pair gets no row."""
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=50, H=256, E=16, R=4, K=2, A=1, router="uniform", seed=4)
    idx = wl.topk_idx.clone()
    idx[7, 1] = 16
    h = ep.ep_handle_create(ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A))
    try:
        fused(h, wl, False, idx_d=idx.to(dev))
        assert ep.ep_get_status(h) & ep.EP_DEV_BAD_EXPERT
        pos = torch.empty((wl.T, wl.K), dtype=torch.int32, device=dev)
        ep.ep_copy_routing(h, pos)
        assert int(pos[7, 1]) == -1
    finally:
        ep.ep_handle_destroy(h)


def test_fused_invalid_id_sets_status():
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=400, H=256, E=16, R=4, K=2, A=1, router="uniform", seed=4)
    idx = wl.topk_idx.clone()
    idx[7, 1] = 16
    h = ep.ep_handle_create(ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A))
    try:
        fused(h, wl, False, idx_d=idx.to(dev))
        assert ep.ep_get_status(h) & ep.EP_DEV_BAD_EXPERT
        pos = torch.empty((wl.T, wl.K), dtype=torch.int32, device=dev)
        ep.ep_copy_routing(h, pos)
        assert int(pos[7, 1]) == -1
    finally:
        ep.ep_handle_destroy(h)


def test_fused_then_plain_dispatch_and_determinism():
    """The handle a fused call filled serves plain dispatches; two fused calls
    give identical bytes."""
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=2500, H=512, E=64, R=8, K=8, A=8, router="group", seed=42)
    o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A, topk_weights=wl.topk_weights.numpy())
    h = ep.ep_handle_create(ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A))
    try:
        outs1, recv1, cap = fused(h, wl, False)
        outs2, recv2, _ = fused(h, wl, False)
        torch.cuda.synchronize()
        assert torch.equal(recv1[0].view(torch.int16), recv2[0].view(torch.int16))
        for k in outs1:
            assert torch.equal(outs1[k], outs2[k]), k
        check_layout(h, wl, outs2, o)
        x2 = workloads.bf16_normal(np.random.default_rng(3), wl.T, wl.H)
        recv = torch.empty((cap, wl.H), dtype=torch.bfloat16, device=dev)
        ep.ep_dispatch(h, x2.to(dev), recv)
        np.testing.assert_array_equal(workloads.bf16_bits(recv[:o.rows]),
                                      oracle.dispatch_bf16(workloads.bf16_bits(x2), o.row_src))
        assert ep.ep_get_status(h) == 0
    finally:
        ep.ep_handle_destroy(h)


def test_fused_lookback_wait_gives_up():
    """The first chunk never publishes its counts (test hook): the look-back
    waits of the chunks after it in its super-chunk run out after 20 ms and
    set EP_DEV_WAIT_TIMEOUT; after ep_clear_status the handle computes the
    right result again."""
    wl = workloads.generate(None, T=4000, H=256, E=64, R=8, K=8, A=2, router="topk", seed=5)
    o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A, topk_weights=wl.topk_weights.numpy())
    h = ep.ep_handle_create(ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A))
    try:
        ep.ep_set_wait_limit(h, 20_000_000, 1)
        fused(h, wl, False)
        assert ep.ep_get_status(h) & ep.EP_DEV_WAIT_TIMEOUT
        ep.ep_set_wait_limit(h, 1_000_000_000, 0)
        ep.ep_clear_status(h)
        outs, recv, cap = fused(h, wl, False)
        assert ep.ep_get_status(h) == 0
        check_layout(h, wl, outs, o)
        check_rows(wl, recv, o, False, cap)
    finally:
        ep.ep_handle_destroy(h)


@pytest.mark.parametrize("T", [3000, 120])
def test_fused_graph_replay(T):
    """Fused layout + dispatch and the combine captured once in a CUDA graph
    and replayed on new routings: the look-back words carry a tag the kernel
    takes from the device each launch, so replays with frozen parameters stay
    correct (T = 3000); the small-batch kernel keeps no state between
    launches (T = 120)."""
    dev = torch.device("cuda")
    base = workloads.generate(None, T=T, H=512, E=64, R=8, K=8, A=4, router="topk", seed=50)
    cfg = ep.make_config(base.T, base.H, base.E, base.R, base.K, base.A)
    cap = ep.ep_capacity_rows(cfg)
    h = ep.ep_handle_create(cfg)
    try:
        idx_d, w_d, x_d = base.topk_idx.to(dev), base.topk_weights.to(dev), base.x.to(dev)
        recv = torch.empty((cap, base.H), dtype=torch.bfloat16, device=dev)
        out = torch.empty((base.T, base.H), dtype=torch.bfloat16, device=dev)
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            ep.ep_layout_dispatch(h, idx_d, w_d, x_d, recv, stream=s)
            ep.ep_combine(h, recv, w_d, out, stream=s)
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            ep.ep_layout_dispatch(h, idx_d, w_d, x_d, recv, stream=s)
            ep.ep_combine(h, recv, w_d, out, stream=s)
        for seed in (51, 52, 53):
            wl = workloads.generate(None, T=T, H=512, E=64, R=8, K=8, A=4, router="topk", seed=seed)
            idx_d.copy_(wl.topk_idx.to(dev))
            w_d.copy_(wl.topk_weights.to(dev))
            x_d.copy_(wl.x.to(dev))
            g.replay()
            torch.cuda.synchronize()
            o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A)
            np.testing.assert_array_equal(workloads.bf16_bits(recv[:o.rows]),
                                          oracle.dispatch_bf16(workloads.bf16_bits(wl.x), o.row_src))
            ref = wl.x.double().numpy() * wl.topk_weights.double().numpy().sum(1, keepdims=True)
            combine_close(out, ref)
        assert ep.ep_get_status(h) == 0
        del g
    finally:
        ep.ep_handle_destroy(h)


def test_fused_empty_batch():
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=0, H=256, E=16, R=4, K=2, A=8, router="topk", seed=1)
    h = ep.ep_handle_create(ep.make_config(0, 256, 16, 4, 2, 8))
    try:
        cnt = torch.full((16,), -9, dtype=torch.int32, device=dev)
        eoff = torch.full((17,), -9, dtype=torch.int32, device=dev)
        x = torch.empty((0, 256), dtype=torch.bfloat16, device=dev)
        ep.ep_layout_dispatch(h, torch.empty((0, 2), dtype=torch.int64, device=dev), None, x, x,
                              num_tokens_per_expert=cnt, expert_offsets=eoff)
        assert ep.ep_get_status(h) == 0 and ep.ep_get_num_rows(h) == 0
        assert (cnt == 0).all() and (eoff == 0).all()
        del wl
    finally:
        ep.ep_handle_destroy(h)
