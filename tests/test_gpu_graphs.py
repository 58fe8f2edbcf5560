"""The normal path captured in a CUDA graph and replayed on new routings.

One capture of ep_get_layout + ep_dispatch + ep_combine (static buffers, the
inputs rewritten in place between replays) must give the oracle's layout and
the identity-expert round trip on every replay -- for a batch that takes the
cluster layout kernel, for one that takes the cooperative kernel, whose
grid-wide wait takes its target from the device (a replayed launch carries the
parameters of the captured one), and for a small batch (fewer than two tokens
per SM) that takes the small-batch layout kernel.
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


SHAPES = [
    dict(T=2048, H=256, E=64, R=8, K=8, A=4, router="topk"),     # cluster layout (8 CTAs)
    dict(T=20000, H=64, E=64, R=8, K=8, A=2, router="topk"),     # cooperative layout (160 000 pairs)
    dict(T=128, H=512, E=256, R=32, K=8, A=2, router="topk"),    # small-batch layout (one CTA per token)
]


@pytest.mark.parametrize("shape", SHAPES, ids=["cluster", "cooperative", "small"])
def test_normal_path_graph_replay(shape):
    dev = torch.device("cuda")
    wls = [workloads.generate(None, seed=70 + i, **shape) for i in range(3)]
    wl0 = wls[0]
    cfg = ep.make_config(wl0.T, wl0.H, wl0.E, wl0.R, wl0.K, wl0.A)
    h = ep.ep_handle_create(cfg)
    try:
        cap = ep.ep_capacity_rows(cfg)
        idx_d, w_d, x_d = wl0.topk_idx.to(dev), wl0.topk_weights.to(dev), wl0.x.to(dev)
        cnt = torch.zeros((wl0.E,), dtype=torch.int32, device=dev)
        rtok = torch.zeros((wl0.R,), dtype=torch.int32, device=dev)
        eoff = torch.zeros((wl0.E + 1,), dtype=torch.int32, device=dev)
        roff = torch.zeros((wl0.R + 1,), dtype=torch.int32, device=dev)
        recv = torch.zeros((cap, wl0.H), dtype=torch.bfloat16, device=dev)
        out = torch.zeros((wl0.T, wl0.H), dtype=torch.bfloat16, device=dev)

        def step():
            ep.ep_get_layout(h, idx_d, w_d, cnt, rtok, None, eoff, roff)
            ep.ep_dispatch(h, x_d, recv)
            ep.ep_combine(h, recv, w_d, out)

        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for wl in wls[1:] + wls[:1] + wls[1:2]:
            idx_d.copy_(wl.topk_idx)
            w_d.copy_(wl.topk_weights)
            x_d.copy_(wl.x)
            out.zero_()
            g.replay()
            torch.cuda.synchronize()
            o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A)
            np.testing.assert_array_equal(cnt.cpu().numpy(), o.num_tokens_per_expert)
            np.testing.assert_array_equal(rtok.cpu().numpy(), o.num_tokens_per_rank)
            np.testing.assert_array_equal(eoff.cpu().numpy(), o.expert_offsets)
            np.testing.assert_array_equal(roff.cpu().numpy(), o.rank_offsets)
            pos = torch.empty((wl.T, wl.K), dtype=torch.int32, device=dev)
            ep.ep_copy_routing(h, pos)
            np.testing.assert_array_equal(pos.cpu().numpy(), o.pos)
            x64 = (workloads.bf16_bits(wl.x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            combine_close(out, x64 * wl.topk_weights.numpy().astype(np.float64).sum(1, keepdims=True))
        del g
        assert ep.ep_get_status(h) == 0
    finally:
        ep.ep_handle_destroy(h)
