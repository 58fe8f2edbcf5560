"""The cross-GPU path of combine_ep_get_08_b200.dist through the CUDA kernels
and NCCL, at the group size one GPU allows (world size 1: the all_to_all
delivers every segment to this rank), and the peer-memory exchange
(dispatch_peer / combine_peer, bf16 and FP8) over the same NCCL group.  The
exchange logic for several ranks is covered over gloo in
test_dist_exchange.py, and the peer exchange across two processes in
test_gpu_peer_ipc.py.
"""
import os
import socket

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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_dispatch_exchange_combine_nccl_one_rank():
    import torch.distributed as dist

    from combine_ep_get_08_b200 import dist as epd
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev)
    try:
        wl = workloads.generate(None, T=512, H=1024, E=32, R=1, K=4, A=8, router="topk", seed=55)
        cfg = ep.make_config(wl.T, wl.H, wl.E, 1, wl.K, wl.A)
        h = ep.ep_handle_create(cfg)
        try:
            cap = ep.ep_capacity_rows(cfg)
            x, idx, w = wl.x.to(dev), wl.topk_idx.to(dev), wl.topk_weights.to(dev)
            send = torch.empty((cap, wl.H), dtype=torch.bfloat16, device=dev)
            recv, plan = epd.dispatch(h, x, idx, w, send, cfg)
            o = oracle.layout(wl.topk_idx.numpy(), wl.E, 1, wl.A)
            assert plan.total_recv == o.rows and plan.total_send == o.rows
            np.testing.assert_array_equal(plan.recv_expert_pairs.numpy().ravel(), o.num_tokens_per_expert)
            np.testing.assert_array_equal(workloads.bf16_bits(recv),
                                          oracle.dispatch_bf16(workloads.bf16_bits(wl.x), o.row_src))
            y_send = torch.empty((cap, wl.H), dtype=torch.bfloat16, device=dev)
            out = torch.empty_like(x)
            epd.combine(h, recv, plan, w, out, y_send)        # identity experts
            torch.cuda.synchronize()
            x64 = (workloads.bf16_bits(wl.x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            combine_close(out, x64 * wl.topk_weights.numpy().astype(np.float64).sum(1, keepdims=True))
            assert ep.ep_get_status(h) == 0

            # the exchange inside the kernels over the same NCCL group: bf16 and FP8
            for fp8 in (False, True):
                bufs = epd.PeerBuffers(max_rows=cap, hidden=wl.H, fp8=fp8)
                try:
                    got, pplan = epd.dispatch_peer(h, x, idx, w, cfg, bufs)
                    assert pplan.recv_rows == [o.rows] and pplan.row0 == [0]
                    xb = workloads.bf16_bits(wl.x)
                    if fp8:
                        q, sc = got
                        oq, osc = oracle.dispatch_fp8(xb, o.row_src)
                        np.testing.assert_array_equal(q.cpu().numpy(), oq)
                        np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), osc.view(np.uint32))
                    else:
                        np.testing.assert_array_equal(workloads.bf16_bits(got), oracle.dispatch_bf16(xb, o.row_src))
                    bufs.y[:pplan.total_recv] = recv               # identity experts
                    out_p = torch.empty_like(x)
                    epd.combine_peer(h, pplan, w, out_p, bufs)
                    assert torch.equal(out_p.view(torch.int16), out.view(torch.int16))
                finally:
                    bufs.close()
            # the same on a caller-given side stream (host reads and collectives
            # must wait for the kernels enqueued there)
            side = torch.cuda.Stream(dev)
            recv2, plan2 = epd.dispatch(h, x, idx, w, send, cfg, stream=side)
            assert plan2.total_recv == o.rows
            np.testing.assert_array_equal(workloads.bf16_bits(recv2), workloads.bf16_bits(recv))
            out2 = torch.empty_like(x)
            epd.combine(h, recv2, plan2, w, out2, y_send, stream=side)
            side.synchronize()
            assert torch.equal(out2.view(torch.int16), out.view(torch.int16))
            bufs = epd.PeerBuffers(max_rows=cap, hidden=wl.H)
            try:
                got, pplan = epd.dispatch_peer(h, x, idx, w, cfg, bufs, stream=side)
                np.testing.assert_array_equal(workloads.bf16_bits(got), workloads.bf16_bits(recv))
                bufs.y[:pplan.total_recv] = recv
                out3 = torch.empty_like(x)
                epd.combine_peer(h, pplan, w, out3, bufs, stream=side)
                assert torch.equal(out3.view(torch.int16), out.view(torch.int16))
            finally:
                bufs.close()
            assert ep.ep_get_status(h) == 0
        finally:
            ep.ep_handle_destroy(h)
    finally:
        dist.destroy_process_group()
