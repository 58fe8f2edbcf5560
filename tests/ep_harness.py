"""Helpers shared by the GPU tests: run the CUDA path through the C ABI and
fetch its results, and compare them with the CPU oracle."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import combine_ep_get_08_b200 as ep
import workloads

RTOL, ATOL = 1e-2, 1e-3   # combine tolerance (fp32 accumulation, bf16 output)
ROW_CHUNK = 16384         # received rows compared per oracle call (bounds host memory)
TOKEN_CHUNK = 2048        # tokens compared per oracle call


def chunks(sel, n):
    """Consecutive slices of at most n entries of sel."""
    for i in range(0, len(sel), n):
        yield sel[i:i + n]


@dataclass
class GpuLayout:
    handle: int
    rows: int
    cap: int
    num_tokens_per_expert: np.ndarray
    num_tokens_per_rank: np.ndarray
    is_token_in_rank: np.ndarray
    expert_offsets: np.ndarray
    rank_offsets: np.ndarray
    pos: np.ndarray
    row_src: np.ndarray
    row_slot: np.ndarray
    row_weight: np.ndarray
    status: int


def config_of(wl) -> ep.ep_config:
    return ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A)


def gpu_layout(wl, idx_d=None, w_d=None, handle=None, with_weights=True) -> GpuLayout:
    dev = torch.device("cuda")
    cfg = config_of(wl)
    h = handle if handle is not None else ep.ep_handle_create(cfg)
    cap = ep.ep_capacity_rows(cfg)
    idx_d = wl.topk_idx.to(dev) if idx_d is None else idx_d
    w_d = (wl.topk_weights.to(dev) if with_weights else None) if w_d is None else w_d
    cnt = torch.full((wl.E,), -9, dtype=torch.int32, device=dev)
    rtok = torch.full((wl.R,), -9, dtype=torch.int32, device=dev)
    in_rank = torch.full((wl.T, wl.R), 7, dtype=torch.uint8, device=dev)
    eoff = torch.full((wl.E + 1,), -9, dtype=torch.int32, device=dev)
    roff = torch.full((wl.R + 1,), -9, dtype=torch.int32, device=dev)
    ep.ep_get_layout(h, idx_d, w_d, cnt, rtok, in_rank, eoff, roff)
    pos = torch.full((wl.T, wl.K), -9, dtype=torch.int32, device=dev)
    src = torch.full((max(cap, 1),), -9, dtype=torch.int32, device=dev)
    slot = torch.full((max(cap, 1),), -9, dtype=torch.int32, device=dev)
    wt = torch.full((max(cap, 1),), -9.0, dtype=torch.float32, device=dev)
    ep.ep_copy_routing(h, pos, src, slot, wt)
    rows = ep.ep_get_num_rows(h)
    status = ep.ep_get_status(h)
    return GpuLayout(h, rows, cap, cnt.cpu().numpy(), rtok.cpu().numpy(), in_rank.cpu().numpy(),
                     eoff.cpu().numpy(), roff.cpu().numpy(), pos.cpu().numpy(),
                     src.cpu().numpy()[:rows], slot.cpu().numpy()[:rows], wt.cpu().numpy()[:rows], status)


LAYOUT_KEYS = ("num_tokens_per_expert", "num_tokens_per_rank", "is_token_in_rank",
               "expert_offsets", "rank_offsets", "pos", "row_src", "row_slot", "row_weight")


def assert_layout_equal(g: GpuLayout, o, with_weights=True):
    assert g.status == 0, f"device status {g.status:#x}"
    assert g.rows == o.rows
    for key in LAYOUT_KEYS:
        if key == "row_weight" and not with_weights:
            continue
        a, b = getattr(g, key), getattr(o, key)
        np.testing.assert_array_equal(a, b.reshape(a.shape), err_msg=key)


def expert_outputs(wl, rows: int, seed: int = 99) -> torch.Tensor:
    """Stand-in expert outputs y [rows, H] bf16 (seeded N(0,1))."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return workloads.bf16_normal(rng, max(rows, 1), wl.H)


def combine_close(out_gpu_bf16: torch.Tensor, ref64: np.ndarray):
    got = out_gpu_bf16.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref64)
    lim = ATOL + RTOL * np.abs(ref64)
    bad = err > lim
    assert not bad.any(), (f"{int(bad.sum())} elements outside rtol={RTOL}, atol={ATOL}; "
                           f"max err {float(err.max()):.3e}")
    return float(err.max())
