"""Parity of ep_dispatch_peer / ep_combine_peer (through the C ABI) with the
CPU oracle, with W ranks' buffers on one GPU and one handle per source rank.

Every source s routes its own tokens over all E experts (num_ranks = W).
Destination r's buffer must hold, for s = 0..W-1 in order, exactly the rows
the oracle lays out for rank r from source s, starting at row0_s[r] =
rows that sources 0..s-1 send to r; rows past them stay untouched.  The FP8
form must write the oracle's E4M3 codes and fp32 scales the same way.  The peer
combine, reading stand-in expert outputs from the W buffers, must equal the
oracle's weighted sum within the combine tolerance, and ep_combine on the
same rows gathered into one local buffer bit for bit (same fp32 order).
"""
import numpy as np
import pytest
import torch

import combine_ep_get_08_b200 as ep
import oracle
import workloads
from ep_harness import combine_close

pytestmark = pytest.mark.gpu

SENTINEL = 12345


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_ep_get_08_b200 import build_lib
    build_lib.build()
    oracle.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _sources(W, T, H, E, K, A, router, seed, idx_edit=None):
    out = []
    for s in range(W):
        wl = workloads.generate(None, T=T, H=H, E=E, R=W, K=K, A=A, router=router, seed=seed + 17 * s)
        if idx_edit is not None:
            wl.topk_idx = idx_edit(wl.topk_idx.clone(), s)
        out.append(wl)
    return out


def run_peer(W, T, H, E, K, A, router="topk", seed=500, idx_edit=None, fp8=False):
    dev = torch.device("cuda")
    wls = _sources(W, T, H, E, K, A, router, seed, idx_edit)
    orc = [oracle.layout(wl.topk_idx.numpy(), E, W, A, topk_weights=wl.topk_weights.numpy()) for wl in wls]
    assert all(o.status == 0 for o in orc)
    S = np.array([np.diff(o.rank_offsets) for o in orc], np.int64)     # S[s, r]
    row0 = np.vstack([np.zeros(W, np.int64), np.cumsum(S, 0)[:-1]])   # row0[s, r]
    recv_total = S.sum(0)
    max_rows = int(recv_total.max()) + 5                               # 5 rows of slack past the blocks
    handles = []
    try:
        for wl in wls:
            h = ep.ep_handle_create(ep.make_config(T, H, E, W, K, A))
            handles.append(h)
            roff = torch.empty(W + 1, dtype=torch.int32, device=dev)
            ep.ep_get_layout(h, wl.topk_idx.to(dev), wl.topk_weights.to(dev), rank_offsets=roff)
            np.testing.assert_array_equal(roff.cpu().numpy(), orc[len(handles) - 1].rank_offsets)
        row0_d = [torch.from_numpy(row0[s].astype(np.int32)).to(dev) for s in range(W)]
        xb = [workloads.bf16_bits(wl.x) for wl in wls]
        if fp8:
            codes = [torch.full((max_rows, H), 0x5A, dtype=torch.uint8, device=dev) for _ in range(W)]
            scales = [torch.full((max_rows, H // 128), -3.0, dtype=torch.float32, device=dev) for _ in range(W)]
            bases = torch.tensor([t.data_ptr() for t in codes], dtype=torch.int64, device=dev)
            sbases = torch.tensor([t.data_ptr() for t in scales], dtype=torch.int64, device=dev)
            for s, (h, wl) in enumerate(zip(handles, wls)):
                ep.ep_dispatch_peer_fp8(h, wl.x.to(dev), bases, sbases, row0_d[s])
            torch.cuda.synchronize()
            ref = [oracle.dispatch_fp8(xb[s], orc[s].row_src) for s in range(W)]
            for r in range(W):
                n = int(recv_total[r])
                segs = [(orc[s].rank_offsets[r], orc[s].rank_offsets[r + 1]) for s in range(W)]
                want_q = np.concatenate([ref[s][0][a:b] for s, (a, b) in enumerate(segs)] + [np.zeros((0, H), np.uint8)])
                want_s = np.concatenate([ref[s][1][a:b] for s, (a, b) in enumerate(segs)]
                                        + [np.zeros((0, H // 128), np.float32)])
                np.testing.assert_array_equal(codes[r][:n].cpu().numpy(), want_q, err_msg=f"codes at rank {r}")
                np.testing.assert_array_equal(scales[r][:n].cpu().numpy().view(np.uint32), want_s.view(np.uint32),
                                              err_msg=f"scales at rank {r}")
                assert bool((codes[r][n:] == 0x5A).all()) and bool((scales[r][n:] == -3.0).all())
            del codes, scales
        else:
            recv = [torch.full((max_rows, H), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
                    for _ in range(W)]
            bases = torch.tensor([t.data_ptr() for t in recv], dtype=torch.int64, device=dev)
            for s, (h, wl) in enumerate(zip(handles, wls)):
                ep.ep_dispatch_peer(h, wl.x.to(dev), bases, row0_d[s])
            torch.cuda.synchronize()
            # destination r: the blocks of sources 0..W-1 in order, then untouched rows
            rows_of = [oracle.dispatch_bf16(xb[s], orc[s].row_src) for s in range(W)]
            for r in range(W):
                want = np.concatenate([rows_of[s][orc[s].rank_offsets[r]:orc[s].rank_offsets[r + 1]]
                                       for s in range(W)] + [np.zeros((0, H), np.uint16)])
                got = workloads.bf16_bits(recv[r])
                n = int(recv_total[r])
                assert n == want.shape[0]
                np.testing.assert_array_equal(got[:n], want, err_msg=f"rows received by rank {r}")
                assert bool((recv[r][n:].view(torch.int16) == SENTINEL).all()), f"rank {r}: rows past the blocks"
            del recv
        # combine: stand-in expert outputs in every rank's buffer (seeded N(0,1))
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed + 1)
        ys = [torch.randn((max_rows, H), generator=gen, device=dev).to(torch.bfloat16) for _ in range(W)]
        y_bases = torch.tensor([t.data_ptr() for t in ys], dtype=torch.int64, device=dev)
        for s, (h, wl, o) in enumerate(zip(handles, wls, orc)):
            w_d = wl.topk_weights.to(dev)
            out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
            ep.ep_combine_peer(h, y_bases, row0_d[s], w_d, out)
            # the same rows gathered into one local buffer in this source's layout
            rows = int(o.rank_offsets[-1])
            y_local = torch.zeros((max(rows, 1), H), dtype=torch.bfloat16, device=dev)
            for r in range(W):
                a, b = int(o.rank_offsets[r]), int(o.rank_offsets[r + 1])
                y_local[a:b] = ys[r][int(row0[s, r]):int(row0[s, r]) + b - a]
            out_local = torch.empty_like(out)
            ep.ep_combine(h, y_local, w_d, out_local)
            assert torch.equal(out.view(torch.int16), out_local.view(torch.int16)), f"source {s}: peer vs local"
            ref = oracle.combine(workloads.bf16_bits(y_local), o.pos, wl.topk_weights.numpy())
            combine_close(out, ref)
        for h in handles:
            assert ep.ep_get_status(h) == 0
    finally:
        for h in handles:
            ep.ep_handle_destroy(h)


CASES = [
    dict(W=2, T=300, H=7168, E=16, K=4, A=1, router="topk", seed=501),
    dict(W=4, T=257, H=200, E=32, K=6, A=3, router="uniform", seed=502),     # ragged row, padding rows
    dict(W=8, T=1000, H=512, E=64, K=8, A=128, router="group", seed=503),    # mostly padding
    dict(W=4, T=1, H=64, E=8, K=2, A=1, router="topk", seed=504),
    dict(W=8, T=2048, H=2048, E=256, K=8, A=1, router="zipf", seed=505),     # skewed ranks
    dict(W=32, T=24, H=128, E=64, K=4, A=2, router="topk", seed=506),        # many ranks, some empty segments
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"W{c['W']}T{c['T']}H{c['H']}E{c['E']}K{c['K']}A{c['A']}")
@pytest.mark.parametrize("fp8", [False, True])
def test_peer_parity(case, fp8):
    if fp8 and case["H"] % 128:
        pytest.skip("FP8 needs H % 128 == 0")
    run_peer(**case, fp8=fp8)


def test_peer_empty_segments_and_masked_slots():
    """Sources that send nothing to some ranks (empty segments), and -1 slots."""
    W, E = 4, 16

    def edit(idx, s):
        idx = idx % 4 + 8 * (idx % 2)          # experts 0-3 (rank 0) and 8-11 (rank 2) only
        idx[torch.arange(idx.shape[0]) % 3 == s % 3, -1] = -1
        idx[0, :] = -1                          # a token with no expert at all
        return idx

    def dedup(idx, s):                          # distinct experts per token, as a router gives
        idx = edit(idx, s)
        for t in range(idx.shape[0]):
            seen = set()
            for k in range(idx.shape[1]):
                v = int(idx[t, k])
                if v >= 0 and v in seen:
                    idx[t, k] = -1
                seen.add(v)
        return idx

    run_peer(W, 120, 256, E, 3, 2, router="topk", seed=510, idx_edit=dedup)
    run_peer(W, 120, 256, E, 3, 2, router="topk", seed=510, idx_edit=dedup, fp8=True)


def test_peer_argument_errors():
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=8, H=64, E=4, R=2, K=2, A=1, router="topk", seed=520)
    h = ep.ep_handle_create(ep.make_config(8, 64, 4, 2, 2, 1))
    try:
        buf = torch.zeros((64, 64), dtype=torch.bfloat16, device=dev)
        bases = torch.tensor([buf.data_ptr()] * 2, dtype=torch.int64, device=dev)
        row0 = torch.zeros(2, dtype=torch.int32, device=dev)
        with pytest.raises(ep.EpError) as e:             # no layout yet
            ep.ep_dispatch_peer(h, wl.x.to(dev), bases, row0)
        assert e.value.code == ep.EP_ERR_STATE
        ep.ep_get_layout(h, wl.topk_idx.to(dev), wl.topk_weights.to(dev))
        with pytest.raises(ep.EpError) as e:
            ep.ep_dispatch_peer(h, wl.x.to(dev), None, row0)
        assert e.value.code == ep.EP_ERR_ARG
        with pytest.raises(ep.EpError) as e:             # misaligned x
            ep.ep_dispatch_peer(h, wl.x.to(dev).view(-1)[1:].data_ptr(), bases, row0)
        assert e.value.code == ep.EP_ERR_ARG
        with pytest.raises(ep.EpError) as e:
            ep.ep_combine_peer(h, bases, row0, None, buf)
        assert e.value.code == ep.EP_ERR_ARG
        with pytest.raises(ep.EpError) as e:             # FP8 needs H % 128 == 0
            ep.ep_dispatch_peer_fp8(h, wl.x.to(dev), bases, bases, row0)
        assert e.value.code == ep.EP_ERR_ARG
    finally:
        ep.ep_handle_destroy(h)


def test_peer_empty_batch_launches_nothing():
    dev = torch.device("cuda")
    h = ep.ep_handle_create(ep.make_config(0, 256, 8, 2, 2, 1))
    try:
        ep.ep_get_layout(h, torch.empty((0, 2), dtype=torch.int64, device=dev))
        buf = torch.zeros((4, 256), dtype=torch.bfloat16, device=dev)
        bases = torch.tensor([buf.data_ptr()] * 2, dtype=torch.int64, device=dev)
        row0 = torch.zeros(2, dtype=torch.int32, device=dev)
        n0 = ep.ep_launch_count()
        ep.ep_dispatch_peer(h, None, bases, row0)
        ep.ep_dispatch_peer_fp8(h, None, bases, bases, row0)
        ep.ep_combine_peer(h, bases, row0, None, None)
        assert ep.ep_launch_count() == n0
        assert bool((buf == 0).all())
    finally:
        ep.ep_handle_destroy(h)


def test_ipc_handle_offset_inside_an_allocation():
    """The handle names the whole allocation; the offset locates the pointer in it."""
    dev = torch.device("cuda")
    t = torch.empty((64, 256), dtype=torch.bfloat16, device=dev)
    hd0, off0 = ep.ep_ipc_get_handle(t)
    hd1, off1 = ep.ep_ipc_get_handle(t[3:])
    assert len(hd0) == ep.EP_IPC_HANDLE_BYTES and hd0 == hd1
    assert off1 - off0 == 3 * 256 * 2 and off0 >= 0
