"""The peer exchange across processes: two ranks (one process each) whose
buffers are mapped into each other with CUDA IPC (ep_ipc_get_handle /
ep_ipc_open_handle), driven by combine_ep_get_08_b200.dist.dispatch_peer /
combine_peer over a gloo group.

Both processes share one GPU here; the kernels never wait on each other
(ranks are ordered by host barriers between launches), so this is the same
program a node with one GPU per rank runs.  Checks: each rank receives,
source by source, exactly the rows the oracle lays out for it (bit for bit);
with experts that double their rows (exact in bf16), each rank's combine
matches the oracle's weighted sum of its own doubled rows; the FP8 dispatch
delivers the oracle's codes and scales the same way.
"""
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads

pytestmark = pytest.mark.gpu

W, T, H, E, K, A = 2, 384, 1024, 16, 4, 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _source(s):
    wl = workloads.generate(None, T=T, H=H, E=E, R=W, K=K, A=A, router="topk", seed=600 + s)
    o = oracle.layout(wl.topk_idx.numpy(), E, W, A, topk_weights=wl.topk_weights.numpy())
    rows = oracle.dispatch_bf16(workloads.bf16_bits(wl.x), o.row_src)
    return wl, o, rows


def _double_bits(bits):
    f = (bits.astype(np.uint32) << 16).view(np.float32) * np.float32(2.0)
    return (f.view(np.uint32) >> 16).astype(np.uint16)   # exact: doubling keeps the low half zero


def _rank_main(rank, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    import combine_ep_get_08_b200 as ep
    from combine_ep_get_08_b200 import dist as epd

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    dist.init_process_group("gloo", rank=rank, world_size=W, timeout=datetime.timedelta(seconds=120))
    res = {}
    bufs = None
    h = None
    try:
        wl, o, rows = _source(rank)
        srcs = [_source(s) for s in range(W)]
        bufs = epd.PeerBuffers(max_rows=W * (T * K + E * (A - 1)), hidden=H)
        h = ep.ep_handle_create(ep.make_config(T, H, E, W, K, A))
        recv, plan = epd.dispatch_peer(h, wl.x.to(dev), wl.topk_idx.to(dev), wl.topk_weights.to(dev),
                                       ep.make_config(T, H, E, W, K, A), bufs)
        want = np.concatenate([r[os_.rank_offsets[rank]:os_.rank_offsets[rank + 1]] for _, os_, r in srcs])
        res["forward"] = bool(np.array_equal(workloads.bf16_bits(recv), want))
        res["recv_rows"] = plan.recv_rows == [int(np.diff(os_.rank_offsets)[rank]) for _, os_, _ in srcs]
        # experts: y = 2 * row, written into this rank's output buffer
        bufs.y[:plan.total_recv] = recv * 2
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        epd.combine_peer(h, plan, wl.topk_weights.to(dev), out, bufs)
        ref = oracle.combine(_double_bits(rows), o.pos, wl.topk_weights.numpy())
        got = out.float().cpu().numpy().astype(np.float64)
        res["combine"] = bool(np.allclose(got, ref, rtol=1e-2, atol=1e-3))
        # the FP8 form into a second set of mapped buffers: codes and scales
        fbufs = epd.PeerBuffers(max_rows=W * (T * K + E * (A - 1)), hidden=H, fp8=True)
        try:
            (q, sc), plan8 = epd.dispatch_peer(h, wl.x.to(dev), wl.topk_idx.to(dev), wl.topk_weights.to(dev),
                                               ep.make_config(T, H, E, W, K, A), fbufs)
            ref = [oracle.dispatch_fp8(workloads.bf16_bits(wl_s.x), os_.row_src) for wl_s, os_, _ in srcs]
            a = [(os_.rank_offsets[rank], os_.rank_offsets[rank + 1]) for _, os_, _ in srcs]
            want_q = np.concatenate([rq[0][lo:hi] for rq, (lo, hi) in zip(ref, a)])
            want_s = np.concatenate([rq[1][lo:hi] for rq, (lo, hi) in zip(ref, a)])
            res["fp8"] = bool(np.array_equal(q.cpu().numpy(), want_q)) and \
                bool(np.array_equal(sc.cpu().numpy().view(np.uint32), want_s.view(np.uint32))) and \
                plan8.recv_rows == plan.recv_rows
        finally:
            dist.barrier()
            fbufs.close()
        res["status"] = ep.ep_get_status(h)
    finally:
        if h is not None:
            ep.ep_handle_destroy(h)
        if bufs is not None:
            dist.barrier()                   # no rank still reads a peer's buffers
            bufs.close()
        dist.destroy_process_group()
    with open(f"{out_path}.{rank}", "w") as f:
        json.dump(res, f)


def test_two_process_peer_exchange(tmp_path):
    from combine_ep_get_08_b200 import build_lib
    build_lib.build()
    oracle.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out = str(tmp_path / "res")
    mp.spawn(_rank_main, args=(_free_port(), out), nprocs=W, join=True)
    for r in range(W):
        assert json.load(open(f"{out}.{r}")) == {"forward": True, "recv_rows": True, "combine": True, "fp8": True,
                                                 "status": 0}
