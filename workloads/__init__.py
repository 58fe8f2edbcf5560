"""Seeded synthetic inputs for the dispatch/combine path.

This module holds no arithmetic of the method (no counting, permuting,
quantising or reducing): it only draws the router's outputs and the hidden
states, deterministically from a seed, in the shapes of the DeepSeek-V3
workloads the pages quote.  Both the CUDA path (through its tests and the
bench) and the CPU oracle consume exactly these arrays.

Workloads (page "blog.hotdry.top ... deepep-expert-parallel-alltoall", first
section: 4096 tokens per batch, hidden 7168, top-4 groups and top-8 experts;
page "lesson14_deepep" section 1(1): 256 routed experts, top-8; same page's
mode table: decode batches of 1..128 tokens):

  tiny    64 x 256,   16 experts / 4 ranks,  top-2 distinct uniform, bf16
  dsv3    4096 x 7168, 256 experts / 8 ranks, group-limited top-8, bf16
  decode  128 x 7168,  256 experts / 32 ranks, plain top-8, FP8 dispatch
  skew    4096 x 7168, 256 experts / 8 ranks, Zipf(1.2) popularity, align 128, FP8
  large   16384 x 7168, 256 experts / 64 ranks, group-limited top-8, align 128,
          FP8 dispatch, one layout reused by 10 dispatch calls

Recipes (stated, since the pages give none):
  x        bf16 of N(0,1) fp32 draws (round to nearest even)
  uniform  K distinct experts uniformly at random; weights softmax(N(0,1) draws)
  topk     logits N(0,1) [T,E], top-K by logit, weights softmax of selected logits
  group    logits N(0,1); 8 groups of E/8; group score = max logit in group;
           keep the 4 best groups; top-K logits inside them; softmax of those
  zipf     expert popularity p ~ (rank+1)^-1.2 over a seeded permutation of
           experts; K draws without replacement (Gumbel top-K of log p);
           weights softmax(N(0,1) draws)
Within a token the K entries are ordered by decreasing score.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

CONFIGS = {
    "tiny": dict(T=64, H=256, E=16, R=4, K=2, A=1, fp8=False, router="uniform", seed=0, reuse=1),
    "dsv3": dict(T=4096, H=7168, E=256, R=8, K=8, A=1, fp8=False, router="group", seed=1, reuse=1),
    "decode": dict(T=128, H=7168, E=256, R=32, K=8, A=1, fp8=True, router="topk", seed=2, reuse=1),
    "skew": dict(T=4096, H=7168, E=256, R=8, K=8, A=128, fp8=True, router="zipf", seed=3, reuse=1),
    "large": dict(T=16384, H=7168, E=256, R=64, K=8, A=128, fp8=True, router="group", seed=4, reuse=10),
}

DESCRIPTIONS = {
    "tiny": "64 tokens x hidden 256 bf16, 16 experts / 4 ranks, top-2 uniform, align 1",
    "dsv3": "DeepSeek-V3 prefill: 4096 tokens x hidden 7168 bf16, 256 experts / 8 ranks, "
            "group-limited top-8 (8 groups, top-4), align 1, bf16 dispatch + combine",
    "decode": "decode: 128 tokens x hidden 7168, 256 experts / 32 ranks, top-8, "
              "FP8 e4m3 1x128 dispatch, bf16 combine",
    "skew": "skewed: 4096 tokens x hidden 7168, 256 experts / 8 ranks, Zipf(1.2) top-8, "
            "align 128, FP8 dispatch",
    "large": "large prefill: 16384 tokens x hidden 7168, 256 experts / 64 ranks, "
             "group-limited top-8, align 128, FP8 dispatch + bf16 combine, layout reused x10",
}


@dataclass
class Workload:
    name: str
    T: int
    H: int
    E: int
    R: int
    K: int
    A: int
    fp8: bool
    reuse: int
    seed: int
    topk_idx: torch.Tensor          # int64 [T, K]
    topk_weights: torch.Tensor      # fp32 [T, K]
    x: torch.Tensor | None = None   # bf16 [T, H]
    extra: dict = field(default_factory=dict)


def _streams(seed: int):
    ss = np.random.SeedSequence(seed)
    sx, sl, sw, sp = ss.spawn(4)
    return (np.random.Generator(np.random.PCG64(sx)), np.random.Generator(np.random.PCG64(sl)),
            np.random.Generator(np.random.PCG64(sw)), np.random.Generator(np.random.PCG64(sp)))


def _softmax_rows(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.float64)
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    return (p / p.sum(axis=1, keepdims=True)).astype(np.float32)


def _top_by_score(scores: np.ndarray, K: int) -> np.ndarray:
    # stable descending order: ties (measure zero for continuous draws) go to the lower id
    order = np.argsort(-scores, axis=1, kind="stable")
    return order[:, :K]


def route(router: str, T: int, E: int, K: int, rng_l, rng_w, rng_p):
    """Return (topk_idx int64 [T,K], topk_weights fp32 [T,K])."""
    if router == "uniform":
        idx = _top_by_score(rng_l.random((T, E)), K)
        w = _softmax_rows(rng_w.standard_normal((T, K)))
    elif router == "topk":
        logits = rng_l.standard_normal((T, E)).astype(np.float32)
        idx = _top_by_score(logits, K)
        w = _softmax_rows(np.take_along_axis(logits, idx, axis=1))
    elif router == "group":
        G, keep = 8, 4
        logits = rng_l.standard_normal((T, E)).astype(np.float32)
        gscore = logits.reshape(T, G, E // G).max(axis=2)
        gkeep = _top_by_score(gscore, keep)
        mask = np.zeros((T, G), dtype=bool)
        np.put_along_axis(mask, gkeep, True, axis=1)
        masked = np.where(np.repeat(mask, E // G, axis=1), logits, -np.inf)
        idx = _top_by_score(masked, K)
        w = _softmax_rows(np.take_along_axis(logits, idx, axis=1))
    elif router == "zipf":
        perm = rng_p.permutation(E)
        p_rank = (np.arange(E, dtype=np.float64) + 1.0) ** -1.2
        p = np.empty(E)
        p[perm] = p_rank / p_rank.sum()
        gumbel = -np.log(-np.log(rng_l.random((T, E))))
        idx = _top_by_score(np.log(p)[None, :] + gumbel, K)
        w = _softmax_rows(rng_w.standard_normal((T, K)))
    else:
        raise ValueError(f"unknown router {router}")
    return idx.astype(np.int64), w.astype(np.float32)


def bf16_normal(rng, T: int, H: int) -> torch.Tensor:
    """bf16 [T,H] rounded (nearest even) from N(0,1) fp32 draws."""
    a = rng.standard_normal((T, H), dtype=np.float32)
    return torch.from_numpy(a).to(torch.bfloat16)


def generate(name: str | None = None, *, seed: int | None = None, with_x: bool = True,
             **override) -> Workload:
    """Build a named workload (optionally overriding any field, e.g. T=..., H=...)."""
    cfg = dict(CONFIGS[name]) if name else {}
    cfg.update(override)
    if seed is not None:
        cfg["seed"] = seed
    for key in ("T", "H", "E", "R", "K"):
        if key not in cfg:
            raise ValueError(f"missing {key}")
    cfg.setdefault("A", 1)
    cfg.setdefault("fp8", False)
    cfg.setdefault("router", "topk")
    cfg.setdefault("seed", 0)
    cfg.setdefault("reuse", 1)
    rng_x, rng_l, rng_w, rng_p = _streams(cfg["seed"])
    idx, w = route(cfg["router"], cfg["T"], cfg["E"], cfg["K"], rng_l, rng_w, rng_p)
    x = bf16_normal(rng_x, cfg["T"], cfg["H"]) if with_x else None
    return Workload(name=name or "custom", T=cfg["T"], H=cfg["H"], E=cfg["E"], R=cfg["R"],
                    K=cfg["K"], A=cfg["A"], fp8=cfg["fp8"], reuse=cfg["reuse"], seed=cfg["seed"],
                    topk_idx=torch.from_numpy(idx), topk_weights=torch.from_numpy(w), x=x)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """View a bf16 tensor's storage as uint16 bit patterns (numpy, CPU)."""
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
