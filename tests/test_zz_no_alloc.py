"""The allocation-free layout (ep_get_layout_noalloc) against ep_get_layout.

Some callers cannot call cudaMalloc where they route tokens (code that must
not trigger a device allocation, runtimes whose device memory comes only from
their own pools, callers with nowhere to keep a handle).  For them the
library has one entry point that writes the layout into caller buffers and
keeps its scratch in a fixed array inside the library.  This test calls it
through the C ABI several times in a row -- on workloads of different shapes,
so each call reuses an array the previous one left dirty -- and checks every
output against the handle-based entry point bit for bit (the layout is
integer data: the tolerance is zero), and the calls that use the array
against the CPU oracle too.  ep_layout_shape confirms which calls run the
cooperative kernel, the one that keeps its scratch in the array.

This file is collected last on purpose, and it also passes alone in a fresh
process.
"""
import numpy as np
import pytest
import torch

import combine_ep_get_08_b200 as ep
import oracle
import workloads
from ep_harness import gpu_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from combine_ep_get_08_b200 import build_lib
    build_lib.build()
    oracle.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def noalloc_layout(wl, with_weights=True):
    dev = torch.device("cuda")
    cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A)
    cap = ep.ep_capacity_rows(cfg)
    i32 = dict(dtype=torch.int32, device=dev)
    out = dict(
        pos=torch.full((wl.T, wl.K), -9, **i32),
        row_src=torch.full((max(cap, 1),), -9, **i32),
        row_slot=torch.full((max(cap, 1),), -9, **i32),
        row_weight=torch.full((max(cap, 1),), -9.0, dtype=torch.float32, device=dev),
        num_tokens_per_expert=torch.full((wl.E,), -9, **i32),
        num_tokens_per_rank=torch.full((wl.R,), -9, **i32),
        is_token_in_rank=torch.full((wl.T, wl.R), 7, dtype=torch.uint8, device=dev),
        expert_offsets=torch.full((wl.E + 1,), -9, **i32),
        rank_offsets=torch.full((wl.R + 1,), -9, **i32),
        status=torch.full((1,), 12345, **i32),
    )
    ep.ep_get_layout_noalloc(cfg, wl.topk_idx.to(dev), wl.topk_weights.to(dev) if with_weights else None,
                             out["pos"], out["row_src"], out["row_slot"],
                             out["row_weight"] if with_weights else None,
                             out["num_tokens_per_expert"], out["num_tokens_per_rank"], out["is_token_in_rank"],
                             out["expert_offsets"], out["rank_offsets"], out["status"])
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    rows = int(res["expert_offsets"][-1])
    for k in ("row_src", "row_slot", "row_weight"):
        res[k] = res[k][:rows]
    res["rows"] = rows
    return res


def handle_layout(wl):
    g = gpu_layout(wl)
    ep.ep_handle_destroy(g.handle)
    return g


KEYS = ("pos", "row_src", "row_slot", "row_weight", "num_tokens_per_expert", "num_tokens_per_rank",
        "is_token_in_rank", "expert_offsets", "rank_offsets")


def assert_same(na, g):
    assert int(na["status"][0]) == 0 and g.status == 0
    assert na["rows"] == g.rows
    for k in KEYS:
        a, b = na[k], getattr(g, k)
        if k == "row_weight":
            np.testing.assert_array_equal(a.view(np.uint32), b.view(np.uint32), err_msg=k)
        else:
            np.testing.assert_array_equal(a, b.reshape(a.shape), err_msg=k)


def uses_scratch(wl) -> bool:
    """Whether the layout of wl runs the cooperative kernel (and so keeps its
    scratch in the fixed array), from the library's own launch plan."""
    cluster, ctas, need = ep.ep_layout_shape(ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A))
    assert ctas >= 1
    assert (need > 0) == (cluster == 0)
    return need > 0


def assert_oracle(na, wl):
    o = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A, topk_weights=wl.topk_weights.numpy())
    assert o.status == 0 and na["rows"] == o.rows
    for k in KEYS:
        a, b = na[k], getattr(o, k)
        np.testing.assert_array_equal(a.reshape(-1), b.reshape(-1), err_msg=f"{k} vs oracle")


def test_matches_handle_layout_calls_in_a_row():
    shapes = [
        (workloads.generate("dsv3", with_x=False), False),              # a thread-block cluster
        (workloads.generate(None, T=700, H=256, E=64, R=8, K=6, A=5,
                            router="topk", seed=77, with_x=False), False),
        (workloads.generate(None, T=20000, H=64, E=64, R=8, K=8, A=3,   # beyond one cluster: the
                            router="topk", seed=78, with_x=False), True),  # cooperative kernel, the array
        (workloads.generate("skew", with_x=False), False),               # expert_alignment 128
        (workloads.generate("decode", with_x=False), False),             # one CTA, no grid-wide wait
        (workloads.generate(None, T=12000, H=64, E=128, R=16, K=8, A=2,  # the array again, other
                            router="group", seed=79, with_x=False), True),  # columns and chunk count
        (workloads.generate("dsv3", seed=11, with_x=False), False),      # back to the first shape
    ]
    for wl, scratch in shapes:
        assert uses_scratch(wl) == scratch
        na = noalloc_layout(wl)
        assert_same(na, handle_layout(wl))
        if scratch:
            assert_oracle(na, wl)


def test_same_call_twice():
    wl = workloads.generate("large", with_x=False)
    assert uses_scratch(wl)                    # 131 072 pairs: the cooperative kernel
    first = noalloc_layout(wl)
    second = noalloc_layout(wl)
    for k in KEYS:
        np.testing.assert_array_equal(first[k], second[k], err_msg=k)
    assert_same(second, handle_layout(wl))
    assert_oracle(second, wl)


def test_rejects_sizes_beyond_the_array():
    dev = torch.device("cuda")
    # 160 000 pairs need the cooperative kernel: 2048 columns x 148 CTAs, about 1.2 MiB of scratch
    cfg = ep.make_config(20000, 256, 1024, 1024, 8, 1)
    idx = torch.zeros((20000, 8), dtype=torch.int64, device=dev)
    t = torch.zeros(20000 * 8 + 4096, dtype=torch.int32, device=dev)
    with pytest.raises(ep.EpError) as ei:
        ep.ep_get_layout_noalloc(cfg, idx, None, t, t, t, None, t, t, None, t, t, t)
    assert ei.value.code == ep.EP_ERR_UNSUPPORTED
    assert "scratch" in str(ei.value)
