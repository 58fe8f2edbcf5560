"""Parity of the fused expert GEMM + combine (ep_expert_combine) with the oracle.

out[t] = bf16(sum_k w[t,k] * act[pos[t,k]] @ W_e^T); compared with the
oracle's fp64 sum within rtol 1e-2 / atol 1e-3 (bf16 inputs, fp32
accumulation in TMEM, fp32 atomic adds, bf16 output).
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


def run_case(wl, I, N, idx=None, check_tokens=None, seed=3):
    dev = torch.device("cuda")
    if idx is not None:
        wl.topk_idx = idx
    g = gpu_layout(wl)
    try:
        assert g.status == 0
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        act = torch.randn((g.cap, I), generator=gen, device=dev).to(torch.bfloat16)
        w = (torch.randn((wl.E, N, I), generator=gen, device=dev) / I ** 0.5).to(torch.bfloat16)
        tw = wl.topk_weights.to(dev)
        acc = torch.full((wl.T, N), 7.0, dtype=torch.float32, device=dev)
        out = torch.empty((wl.T, N), dtype=torch.bfloat16, device=dev)
        ep.ep_expert_combine(g.handle, act, I, w, N, tw, acc, out)
        torch.cuda.synchronize()
        assert ep.ep_get_status(g.handle) == 0
        o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A)
        sel = None if check_tokens is None else np.asarray(check_tokens, np.int32)
        ref = oracle.expert_combine(workloads.bf16_bits(act[:max(g.rows, 1)]), workloads.bf16_bits(w),
                                    wl.topk_idx.numpy(), o.pos, wl.topk_weights.numpy(), sel)
        got = out if sel is None else out[torch.from_numpy(sel).long().to(dev)]
        combine_close(got, ref)
        return out
    finally:
        ep.ep_handle_destroy(g.handle)


def test_small_one_tile_column():
    wl = workloads.generate(None, T=256, H=128, E=8, R=2, K=4, A=128, router="topk", seed=91)
    run_case(wl, I=128, N=256)


def test_many_tiles_persistent():
    """More tiles than SMs: ring stages and both TMEM accumulators are reused."""
    wl = workloads.generate(None, T=2048, H=128, E=16, R=4, K=8, A=128, router="topk", seed=92)
    run_case(wl, I=512, N=1024, check_tokens=np.r_[0:64, 2000:2048])


def test_masked_slots_and_skew():
    wl = workloads.generate(None, T=512, H=128, E=32, R=8, K=6, A=256, router="zipf", seed=93)
    idx = wl.topk_idx.clone()
    idx[torch.rand(idx.shape, generator=torch.Generator().manual_seed(2)) < 0.2] = -1
    run_case(wl, I=256, N=512, idx=idx)


def test_bench_shape():
    """The shape the bench times: one expert-parallel rank of a DeepSeek-V3
    layer (32 local experts, 4096 tokens x top-8, alignment 128), inner 2048
    -> 7168 outputs: 32-deep k-block accumulation over 28 column blocks and
    ~288 row tiles.  256 tokens (both ends and a seeded sample), all 7168
    columns each, against the oracle."""
    wl = workloads.generate(None, T=4096, H=7168, E=32, R=8, K=8, A=128, router="topk", seed=5, with_x=False)
    rng = np.random.default_rng(17)
    tok = np.unique(np.concatenate([np.arange(32), np.arange(4064, 4096), rng.integers(32, 4064, 200)]))
    run_case(wl, I=2048, N=7168, check_tokens=tok, seed=5)


def test_rejects_unaligned_experts():
    dev = torch.device("cuda")
    wl = workloads.generate(None, T=64, H=128, E=8, R=2, K=2, A=64, router="topk", seed=94)
    g = gpu_layout(wl)
    try:
        act = torch.zeros((g.cap, 128), dtype=torch.bfloat16, device=dev)
        w = torch.zeros((8, 256, 128), dtype=torch.bfloat16, device=dev)
        acc = torch.zeros((64, 256), dtype=torch.float32, device=dev)
        out = torch.zeros((64, 256), dtype=torch.bfloat16, device=dev)
        with pytest.raises(ep.EpError) as e:
            ep.ep_expert_combine(g.handle, act, 128, w, 256, wl.topk_weights.to(dev), acc, out)
        assert e.value.code == ep.EP_ERR_ARG
    finally:
        ep.ep_handle_destroy(g.handle)
