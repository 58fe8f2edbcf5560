#!/usr/bin/env python
"""Benchmark of the dispatch/combine hot path on B200.

One step = layout (ep_get_layout) + dispatch (ep_dispatch, or
ep_dispatch_fp8) + combine (ep_combine) over one batch of the named
workload, through the C ABI.  Default workload: the DeepSeek-V3 prefill
shape (4096 tokens x hidden 7168 bf16, 256 experts over 8 logical ranks,
group-limited top-8), bf16 dispatch + combine, identity experts (combine
reads the dispatched rows).

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and torch.cuda.synchronize() on both sides, timed with CUDA events on the
stream the kernels are launched on.  The 126 MB L2 is flushed (a 256 MiB
read, outside the events: it leaves no dirty lines for the timed kernel to
write back) before each step and between dispatch and combine, where the
expert GEMMs would run.  Layout and dispatch run back to back (the dispatch
launch overlaps the layout's end) and are timed as one span; a separate pass
with an event between them gives each kernel's own time for the breakdown
and the roofline.  value = algorithmic bytes of dispatch + combine per step /
device time of the step, summed over ranks and divided by the max over ranks.
e2e: the same steps with their inputs uploaded from and outputs downloaded
to pinned host memory, pipelined over two buffer slots.

--impl reference times the CPU oracle (single thread) on a bounded sample of
the same workload instead.  --expert-gemm times the expert GEMM with the
fused combine (ep_expert_combine) in TFLOP/s.  --mode ll uses the
low-latency static layout.  Multi-GPU (torchrun): every rank runs its own
replica on its own GPU (independent batches, no collective on the data
path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dispatch+combine µs/call and effective HBM GB/s (% of B200 peak) at 1 GPU"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0          # the B200 specification figure (~8 TB/s)
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------
# byte model (algorithmic bytes, metadata excluded)
# ----------------------------------------------------------------------------
def row_bytes(H: int, fp8: bool) -> int:
    return H + 4 * (H // 128) if fp8 else 2 * H


def dispatch_bytes(T, H, K, rows, fp8) -> int:
    """read x once + write every received row (padding rows included)."""
    return 2 * T * H + rows * row_bytes(H, fp8)


def combine_bytes(T, H, K) -> int:
    """read the T*K expert-output rows (bf16) + write out (bf16)."""
    return 2 * T * K * H + 2 * T * H


# ----------------------------------------------------------------------------
# distributed plumbing (host logic; tested with gloo on CPU)
# ----------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------------------
# clocks (NVML reads only; no setting is changed)
# ----------------------------------------------------------------------------
class ClockSampler:
    REASONS = {  # NVML clocks-event reason bits
        0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
        0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._nvml = None

    def _sample(self):
        nv = self._nvml
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for b, name in self.REASONS.items():
                if bits & b:
                    self.reasons.add(name)
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml is not None:
            # a short region (tens of ms) would otherwise see the sampling
            # thread only at the interpreter's default 5 ms switch interval
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(self.period / 4)
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
            self._sample()
            sys.setswitchinterval(self._switch)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# roofline inputs
# ----------------------------------------------------------------------------
def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


# the sources of the step's kernels (layout, dispatch, combine) and their shared header
STEP_KERNEL_SOURCES = ("combine.cu", "dispatch.cu", "dispatch_lb.cu", "ep_internal.cuh", "fp8_block.cuh", "layout.cu")


def kernel_source_digest() -> str:
    """Digest of the step kernels' code: comments and blank lines are left out,
    so that a comment edit does not invalidate the recorded DRAM traffic."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "combine_ep_get_08_b200", "csrc")
    for name in STEP_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
        h.update(name.encode() + "\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


def ncu_traffic(role: str, workload: str):
    """(kernel name, DRAM bytes per launch) of a role ("layout", "dispatch",
    "combine") from the committed ncu summary, if it was taken on the current
    kernel sources; else (None, None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            data = json.load(f)
    except Exception:  # noqa: BLE001
        return None, None
    if data.get("source_digest") != kernel_source_digest():
        return None, None
    entry = data.get("roles", {}).get(workload, {}).get(role)
    if entry is None:
        return None, None
    return entry.get("kernel"), entry.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------
# CPU oracle arm
# ----------------------------------------------------------------------------
def oracle_sample(wl, budget_s: float, min_steps: int = 1):
    """Time the oracle on full steps of the workload until budget_s elapsed.
    Returns (GB/s, steps, seconds, bytes_per_step)."""
    import numpy as np

    import oracle
    import workloads
    oracle.build()
    idx, w = wl.topk_idx.numpy(), wl.topk_weights.numpy()
    xb = workloads.bf16_bits(wl.x)
    n, t0 = 0, time.perf_counter()
    bytes_step = None
    while True:
        lay = oracle.layout(idx, wl.E, wl.R, wl.A, topk_weights=w)
        if wl.fp8:
            oracle.dispatch_fp8(xb, lay.row_src)
            y = np.zeros((lay.rows, wl.H), np.uint16)
        else:
            y = oracle.dispatch_bf16(xb, lay.row_src)
        oracle.combine(y, lay.pos, w)
        n += 1
        bytes_step = dispatch_bytes(wl.T, wl.H, wl.K, lay.rows, wl.fp8) + combine_bytes(wl.T, wl.H, wl.K)
        el = time.perf_counter() - t0
        if n >= min_steps and el >= budget_s:
            break
    return bytes_step * n / el / 1e9, n, el, bytes_step


def run_reference(args, world, rank):
    import workloads
    if rank != 0:
        return 0
    wl = workloads.generate(args.config)
    _, _, _, bytes_step = oracle_sample(wl, 0.0)              # one untimed call
    # warm-up steps (untimed), then K timed steps; a step is one oracle pass
    # over a token sample of the batch, scaled to GB/s by the bytes it covers
    sample_T = min(wl.T, args.ref_tokens)
    sub = workloads.generate(args.config) if sample_T == wl.T else _subsample(wl, sample_T)
    for _ in range(args.warmup):
        oracle_sample(sub, 0.0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        gbs, _, _, bstep = oracle_sample(sub, 0.0)
    el = time.perf_counter() - t0
    value = bstep * args.steps / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workloads.DESCRIPTIONS[args.config], "sample_tokens": sample_T},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: oracle layout + dispatch + combine over the first "
                                   f"{sample_T} of {wl.T} tokens of the workload (single thread)",
                         "host": host_cpu()},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _subsample(wl, T):
    import copy
    sub = copy.copy(wl)
    sub.T = T
    sub.topk_idx = wl.topk_idx[:T].contiguous()
    sub.topk_weights = wl.topk_weights[:T].contiguous()
    sub.x = wl.x[:T].contiguous()
    return sub


# ----------------------------------------------------------------------------
# CUDA arm
# ----------------------------------------------------------------------------
class Path:
    """Device buffers and one handle for a workload; step() enqueues one pass."""

    def __init__(self, wl, dev):
        import torch

        import combine_ep_get_08_b200 as ep
        self.ep, self.torch, self.wl, self.dev = ep, torch, wl, dev
        cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A)
        self.cap = ep.ep_capacity_rows(cfg)
        self.h = ep.ep_handle_create(cfg)
        self.idx = wl.topk_idx.to(dev)
        self.w = wl.topk_weights.to(dev)
        self.x = wl.x.to(dev)
        if wl.fp8:
            self.recv = torch.empty((self.cap, wl.H), dtype=torch.uint8, device=dev)
            self.scales = torch.empty((self.cap, wl.H // 128), dtype=torch.float32, device=dev)
            g = torch.Generator(device=dev)
            g.manual_seed(7)
            self.y = torch.randn((self.cap, wl.H), generator=g, device=dev).to(torch.bfloat16)
        else:
            self.recv = torch.empty((self.cap, wl.H), dtype=torch.bfloat16, device=dev)
            self.scales = None
            self.y = self.recv                     # identity experts
        self.out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
        # fp32 so that the reduction reads it in place (an int32 sum would first
        # widen it to an int64 copy: 512 MB of writes)
        self.flush_buf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.flush_sink = None

    def flush_l2(self):
        # read 256 MiB (2x the L2): evicts every line without leaving dirty
        # lines behind for the next timed kernel to write back
        self.flush_sink = self.flush_buf.sum()

    def layout(self, stream, idx=None, w=None):
        self.ep.ep_get_layout(self.h, self.idx if idx is None else idx, self.w if w is None else w, stream=stream)

    def dispatch(self, stream, x=None, idx=None):
        x = self.x if x is None else x
        if self.wl.fp8:
            self.ep.ep_dispatch_fp8(self.h, x, self.recv, self.scales, stream=stream)
        else:
            self.ep.ep_dispatch(self.h, x, self.recv, stream=stream)

    def combine(self, stream, out=None, w=None):
        self.ep.ep_combine(self.h, self.y, self.w if w is None else w, self.out if out is None else out,
                           stream=stream)

    def close(self):
        self.ep.ep_handle_destroy(self.h)


class LLPath(Path):
    """The low-latency static layout: M fixed slots per expert, layout fused
    into the dispatch launch (ep_ll_dispatch), no padding rows."""

    def __init__(self, wl, dev, M):
        import torch

        import combine_ep_get_08_b200 as ep
        self.ep, self.torch, self.wl, self.dev = ep, torch, wl, dev
        cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, 1)
        self.M = M
        self.cap = ep.ep_ll_capacity_rows(cfg, M)
        self.h = ep.ep_ll_handle_create(cfg, M)
        self.idx = wl.topk_idx.to(dev)
        self.w = wl.topk_weights.to(dev)
        self.x = wl.x.to(dev)
        self.cnt = torch.zeros((wl.E,), dtype=torch.int32, device=dev)
        if wl.fp8:
            self.recv = torch.empty((self.cap, wl.H), dtype=torch.uint8, device=dev)
            self.scales = torch.empty((ep.ep_ll_scale_buffer_floats(cfg, M),), dtype=torch.float32, device=dev)
            g = torch.Generator(device=dev)
            g.manual_seed(7)
            self.y = torch.randn((self.cap, wl.H), generator=g, device=dev).to(torch.bfloat16)
        else:
            self.recv = torch.empty((self.cap, wl.H), dtype=torch.bfloat16, device=dev)
            self.scales = None
            self.y = self.recv
        self.out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
        self.flush_buf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.flush_sink = None

    def layout(self, stream, idx=None, w=None):
        pass                                   # fused into the dispatch launch

    def dispatch(self, stream, x=None, idx=None):
        x = self.x if x is None else x
        idx = self.idx if idx is None else idx
        if self.wl.fp8:
            self.ep.ep_ll_dispatch_fp8(self.h, idx, x, self.recv, self.scales, self.cnt, stream=stream)
        else:
            self.ep.ep_ll_dispatch(self.h, idx, x, self.recv, self.cnt, stream=stream)

    def combine(self, stream, out=None, w=None):
        self.ep.ep_ll_combine(self.h, self.y, self.w if w is None else w, self.out if out is None else out,
                              stream=stream)


class FusedPath(Path):
    """Layout and the step's first dispatch in one call (ep_layout_dispatch:
    a counts pre-pass, then the dispatch ranks its chunks and places them by
    decoupled look-back); later dispatches of the step reuse the handle."""

    def __init__(self, wl, dev):
        super().__init__(wl, dev)
        self._pending = None

    def layout(self, stream, idx=None, w=None):
        self._pending = (self.idx if idx is None else idx, self.w if w is None else w)

    def dispatch(self, stream, x=None, idx=None):
        if self._pending is None:
            return super().dispatch(stream, x=x)
        x = self.x if x is None else x
        idx, w = self._pending
        self._pending = None
        if self.wl.fp8:
            self.ep.ep_layout_dispatch_fp8(self.h, idx, w, x, self.recv, self.scales, stream=stream)
        else:
            self.ep.ep_layout_dispatch(self.h, idx, w, x, self.recv, stream=stream)


def make_path(name, mode, dev, rank, ll_slots=0):
    """The named workload (rank-seeded) and its device buffers and handle."""
    import workloads
    base = workloads.CONFIGS[name]
    wl = workloads.generate(name, seed=base["seed"] + 1000 * rank)
    if mode == "ll":
        path = LLPath(wl, dev, ll_slots or max(wl.T, 1))
    elif mode == "fused":
        path = FusedPath(wl, dev)
    else:
        path = Path(wl, dev)
    return wl, path


def step_fn(path, reuse, sptr, stream):
    """One step: flush, layout, then `reuse` dispatch/flush/combine calls.
    ev: 5 events (before the layout, unused, after the first dispatch, after
    the flush that follows it, after the first combine); sp: the stream to
    launch on (the bench's stream unless being captured)."""
    def one_step(ev=None, sp=None):
        # The dispatch follows the layout with no event between them, so its
        # launch overlaps the layout's tail (programmatic dependent launch).
        sp = sptr if sp is None else sp
        path.flush_l2()
        if ev is not None:
            ev[0].record(stream)
        path.layout(sp)
        for r in range(reuse):
            path.dispatch(sp)
            if ev is not None and r == 0:
                ev[2].record(stream)
            path.flush_l2()
            if ev is not None and r == 0:
                ev[3].record(stream)
            path.combine(sp)
            if ev is not None and r == 0:
                ev[4].record(stream)
    return one_step


def split_pass(path, n, stream, sptr):
    """Each kernel timed alone (events between layout, dispatch and combine),
    and the L2 write-back each one leaves behind: the 256 MiB read flush that
    follows a kernel also writes back the dirty lines the kernel left in L2,
    so (flush after the kernel) - (flush of a clean L2) is the time of that
    write-back, charged to the kernel in `with_writeback`."""
    import torch
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(10)] for _ in range(n)]
    for e in evs:
        e[0].record(stream)
        path.flush_l2()
        e[1].record(stream)
        path.layout(sptr)
        e[2].record(stream)
        path.dispatch(sptr)
        e[3].record(stream)
        path.flush_l2()                     # writes back what the dispatch left dirty
        e[4].record(stream)
        path.combine(sptr)
        e[5].record(stream)
        path.flush_l2()                     # writes back what the combine left dirty
        e[6].record(stream)
        path.flush_l2()                     # a clean L2: the flush alone
        e[7].record(stream)
        path.dispatch(sptr)                 # a further dispatch on the same layout (handle reuse)
        e[8].record(stream)
        path.flush_l2()
        e[9].record(stream)
    torch.cuda.synchronize()
    el = lambda e, i, j: e[i].elapsed_time(e[j])  # noqa: E731
    return {"layout": [el(e, 1, 2) for e in evs], "dispatch": [el(e, 2, 3) for e in evs],
            "combine": [el(e, 4, 5) for e in evs], "flush_after_dispatch": [el(e, 3, 4) for e in evs],
            "flush_after_combine": [el(e, 5, 6) for e in evs], "flush_clean": [el(e, 6, 7) for e in evs],
            "dispatch_reuse": [el(e, 7, 8) for e in evs]}


def kernel_figures(wl, rows, split, ll, peak):
    """Per-kernel means, GB/s and roofline fractions (of the measured peak and
    of the 8 TB/s B200 figure), plain and with the L2 write-back charged."""
    b_dis = dispatch_bytes(wl.T, wl.H, wl.K, rows, wl.fp8)
    b_com = combine_bytes(wl.T, wl.H, wl.K)
    mean = {k: statistics.mean(v) * 1e3 for k, v in split.items()}      # µs (dispatch_reuse: reported)
    lay = 0.0 if ll else mean["layout"]
    wb_dis = max(0.0, mean["flush_after_dispatch"] - mean["flush_clean"])
    wb_com = max(0.0, mean["flush_after_combine"] - mean["flush_clean"])
    out = {
        "us_per_call": {"layout": round(lay, 2), "dispatch": round(mean["dispatch"], 2),
                        "combine": round(mean["combine"], 2),
                        "dispatch_on_reused_layout": round(mean.get("dispatch_reuse", mean["dispatch"]), 2)},
        "bytes_per_call": {"dispatch": b_dis, "combine": b_com},
        "gbs_per_call": {"dispatch": round(b_dis / mean["dispatch"] / 1e3, 1),
                         "combine": round(b_com / mean["combine"] / 1e3, 1)},
        "frac_of_measured": {"dispatch": round(b_dis / mean["dispatch"] / 1e3 / peak, 4),
                             "combine": round(b_com / mean["combine"] / 1e3 / peak, 4)},
        "frac_of_8tbs": {"dispatch": round(b_dis / mean["dispatch"] / 1e3 / SPEC_HBM_GBS, 4),
                         "combine": round(b_com / mean["combine"] / 1e3 / SPEC_HBM_GBS, 4)},
        "with_writeback": {
            "dispatch_us": round(mean["dispatch"] + wb_dis, 2), "combine_us": round(mean["combine"] + wb_com, 2),
            "dispatch_gbs": round(b_dis / (mean["dispatch"] + wb_dis) / 1e3, 1),
            "combine_gbs": round(b_com / (mean["combine"] + wb_com) / 1e3, 1),
            "dispatch_frac": round(b_dis / (mean["dispatch"] + wb_dis) / 1e3 / peak, 4),
            "combine_frac": round(b_com / (mean["combine"] + wb_com) / 1e3 / peak, 4),
            "flush_clean_us": round(mean["flush_clean"], 2),
            "how": "kernel time + (256 MiB read flush right after the kernel - the same flush of a clean L2): "
                   "the write-back of the lines the kernel left dirty in L2"},
        "us_p10_p50_p90": {k: pct(split[k]) for k in ("layout", "dispatch", "combine")},
    }
    return out


def config_summary(name, mode, args, dev, rank, stream, peak, steps, warmup):
    """One workload measured on its own (no barrier, this rank only): the
    step as `value` times it, per-kernel times with and without the L2
    write-back, and for latency-bound steps the CUDA-graph replay."""
    import torch

    import combine_ep_get_08_b200 as ep
    import workloads
    ll = mode in ("ll", "fused")        # no separate layout launch
    wl, path = make_path(name, mode, dev, rank)
    try:
        reuse = wl.reuse
        sptr = stream.cuda_stream
        one_step = step_fn(path, reuse, sptr, stream)
        for _ in range(warmup):
            one_step()
        torch.cuda.synchronize()
        rows = int(path.cnt.sum()) if isinstance(path, LLPath) else ep.ep_get_num_rows(path.h)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        for e in evs:
            one_step(e)
        torch.cuda.synchronize()
        ld_ms = [e[0].elapsed_time(e[2]) for e in evs]
        com_ms = [e[3].elapsed_time(e[4]) for e in evs]
        split = split_pass(path, steps, stream, sptr)
        fig = kernel_figures(wl, rows, split, ll, peak)
        mean_dis = statistics.mean(split["dispatch_reuse"])   # the step's further dispatches reuse the layout
        step_ms = statistics.mean([ld + (reuse - 1) * mean_dis + reuse * c for ld, c in zip(ld_ms, com_ms)])
        bytes_step = reuse * (fig["bytes_per_call"]["dispatch"] + fig["bytes_per_call"]["combine"])
        entry = {"workload": workloads.DESCRIPTIONS[name] + MODE_NOTE[mode],
                 "steps": steps, "rows": rows, "reuse": reuse,
                 "step_us": round(step_ms * 1e3, 2), "step_gbs": round(bytes_step / (step_ms * 1e-3) / 1e9, 1),
                 "us_layout_then_dispatch": round(statistics.mean(ld_ms) * 1e3, 2)}
        entry.update(fig)
        if bytes_step < L2_FLUSH_BYTES // 8:
            entry["graph"] = run_graph(path, one_step, args, stream, reuse, 1, dev, bytes_step)
        entry["device_status"] = int(ep.ep_get_status(path.h))
        return entry
    finally:
        path.close()


PER_CONFIG = (("dsv3", "fused"), ("tiny", "normal"), ("decode", "normal"), ("decode", "ll"), ("decode", "fused"),
              ("skew", "normal"), ("skew", "fused"), ("large", "normal"), ("large", "fused"))
MODE_NOTE = {"normal": "", "ll": " (low-latency static layout)",
             "fused": " (layout fused into the dispatch: ep_layout_dispatch)"}


def run_cuda(args, world, rank, local):
    import torch

    import combine_ep_get_08_b200 as ep
    import workloads

    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}), flush=True)
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    from combine_ep_get_08_b200 import build_lib
    if rank == 0:
        build_lib.build()
    barrier(world)
    ep.library()

    ll = args.mode in ("ll", "fused")   # no separate layout launch
    wl, path = make_path(args.config, args.mode, dev, rank, args.ll_slots)
    reuse = wl.reuse if args.reuse is None else args.reuse
    if args.sm_limit:
        ep.ep_set_sm_limit(path.h, args.sm_limit)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    one_step = step_fn(path, reuse, sptr, stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    rows = int(path.cnt.sum()) if isinstance(path, LLPath) else ep.ep_get_num_rows(path.h)
    status = ep.ep_get_status(path.h)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    bracket = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    launches0 = ep.ep_launch_count()
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        bracket[0].record(stream)
        for i in range(args.steps):
            one_step(evs[i])
        bracket[1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    launches = ep.ep_launch_count() - launches0

    bracket_ms = bracket[0].elapsed_time(bracket[1])
    # layout + first dispatch as one span (their launches overlap); with
    # reuse > 1 only the first dispatch/combine pair of a step carries events
    # and the further calls count at the per-call time measured below
    ld_ms = [e[0].elapsed_time(e[2]) for e in evs]
    com_ms = [e[3].elapsed_time(e[4]) for e in evs]

    # per-kernel times (events between the kernels) and the L2 write-back
    # each leaves, for the breakdown and the roofline; not part of `value`
    split = split_pass(path, min(args.steps, 20), stream, sptr)
    peak, peak_src = measured_peak()
    fig = kernel_figures(wl, rows, split, ll, peak)
    mean_dis = statistics.mean(split["dispatch_reuse"])   # the step's further dispatches reuse the layout
    step_ms = [ld + (reuse - 1) * mean_dis + reuse * c for ld, c in zip(ld_ms, com_ms)]
    total_ms = sum(step_ms)

    b_dis, b_com = fig["bytes_per_call"]["dispatch"], fig["bytes_per_call"]["combine"]
    bytes_step = reuse * (b_dis + b_com)
    my_bytes = bytes_step * args.steps
    all_bytes = sum_over_ranks(my_bytes, world, dev)
    max_total_ms = max_over_ranks(total_ms, world, dev)
    value = all_bytes / (max_total_ms * 1e-3) / 1e9

    # e2e: same step through the public API with pinned host buffers
    e2e = run_e2e(path, args, stream, reuse, world, dev, bytes_step)
    # latency-bound steps only: for a large step the flush inside the graph
    # also writes back the dispatch's dirty lines, which a flush timed alone
    # does not, so the subtraction would under-correct
    small = bytes_step < L2_FLUSH_BYTES // 8
    graph = run_graph(path, one_step, args, stream, reuse, world, dev, bytes_step) if small else None

    kern = fig["us_per_call"]
    dom = "dispatch" if kern["dispatch"] >= kern["combine"] else "combine"
    dom_bytes = b_dis if dom == "dispatch" else b_com
    achieved = dom_bytes / (kern[dom] * 1e-6) / 1e9
    wb = fig["with_writeback"]
    kname, traffic = ncu_traffic(dom, args.config + ("" if args.mode == "normal" else "-" + args.mode))
    clocks = sampler.summary()
    status_end = ep.ep_get_status(path.h)
    path.close()

    per_config = None
    if world == 1 and not args.no_per_config and args.config == "dsv3" and args.mode == "normal" \
            and not args.sm_limit:
        n = max(5, min(args.steps, 20))
        per_config = {}
        for name, mode in PER_CONFIG:
            per_config[name + ("" if mode == "normal" else "_" + mode)] = config_summary(
                name, mode, args, dev, rank, stream, peak, n, args.warmup)
        # the expert GEMM with the fused combine, both operand types (tensor-bound)
        flush_g = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        for fp8 in (False, True):
            o = expert_gemm_inputs(dev, fp8, rank)
            ms = time_expert_gemm(o, n, args.warmup, flush_g, stream)
            entry = expert_gemm_summary(o, ms)
            entry["device_status"] = int(ep.ep_get_status(o["h"]))
            per_config["expert_gemm_" + ("e4m3" if fp8 else "bf16")] = entry
            ep.ep_handle_destroy(o["h"])
            del o
        del flush_g
        torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(max_total_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {
                "workload": workloads.DESCRIPTIONS[args.config], "name": args.config,
                "rows": rows, "reuse": reuse,
                "layout_mode": {"ll": f"low-latency static: {getattr(path, 'M', 0)} slots per expert, layout "
                                      "fused into the dispatch launch",
                                "fused": "normal padded expert-major rows; layout and dispatch in one call "
                                         "(counts pre-pass + dispatch with decoupled look-back)",
                                "normal": "normal: padded expert-major rows (ep_get_layout, then ep_dispatch)"}[args.mode],
                "parallelism": f"replicas x{world} (independent batches, no data-path collective)",
                "sm_limit": args.sm_limit or None,
                "l2": "flushed (256 MiB read, outside the timed events) before each step and "
                      "between dispatch and combine",
            },
            "us_per_call": kern,
            "us_layout_then_dispatch": round(statistics.mean(ld_ms) * 1e3, 2),
            "us_p10_p50_p90": dict(fig["us_p10_p50_p90"], layout_then_dispatch=pct(ld_ms)),
            "bytes_per_call": fig["bytes_per_call"],
            "gbs_per_call": fig["gbs_per_call"],
            "frac_of_8tbs": fig["frac_of_8tbs"],
            "roofline": {"bound": "hbm", "kernel": dom if kname is None else f"{dom}: {kname}",
                         "achieved": round(achieved, 1), "peak": peak, "peak_source": peak_src,
                         "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                         "with_writeback": {"us": wb[dom + "_us"], "achieved": wb[dom + "_gbs"],
                                            "frac": wb[dom + "_frac"], "how": wb["how"]}},
            "with_writeback": wb,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "clocks": clocks,
            "bracket_ms": round(bracket_ms, 3),
            "device_status": int(status | status_end),
        }
        if graph is not None:
            line["graph"] = graph
        if per_config is not None:
            line["per_config"] = per_config
        if world == 1 and not args.no_cpu_baseline:
            gbs, n, el, _ = oracle_sample(wl, args.cpu_budget)
            line["cpu_baseline"] = {
                "value": round(gbs, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                "sample": f"{n} full step(s) of the same workload (layout + dispatch + combine, "
                          f"{el:.1f} s, single thread)", "host": host_cpu()}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def pct(ms_list) -> list:
    """10th, 50th and 90th percentile of event times in ms, as µs."""
    v = sorted(ms_list)
    if not v:
        return [None, None, None]
    at = lambda q: v[min(len(v) - 1, int(round(q * (len(v) - 1))))]  # noqa: E731
    return [round(at(q) * 1e3, 2) for q in (0.1, 0.5, 0.9)]


def host_cpu() -> dict:
    """The host the oracle baseline ran on: CPU model and logical CPUs."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def run_graph(path, one_step, args, stream, reuse, world, dev, bytes_step):
    """The same step (L2 flushes included) captured once in a CUDA graph and
    replayed: the launch gaps between the kernels mostly disappear, as in a
    serving engine that replays its decode step.  Reported beside `value`,
    which stays the event-timed figure; the flushes are outside `value`'s
    events but inside this span, so their time (measured alone) is taken off."""
    import torch
    n = max(5, min(args.steps, 30))
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        one_step(sp=side.cuda_stream)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        one_step(sp=side.cuda_stream)
    fl = torch.cuda.CUDAGraph()
    with torch.cuda.graph(fl, stream=side):
        path.flush_l2()
        path.flush_l2()
    for _ in range(2):
        g.replay()
        fl.replay()
    torch.cuda.synchronize()
    t = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    barrier(world)
    t[0].record(stream)
    for _ in range(n):
        g.replay()
    t[1].record(stream)
    for _ in range(n):
        fl.replay()
    t[2].record(stream)
    torch.cuda.synchronize()
    ms = (t[0].elapsed_time(t[1]) - t[1].elapsed_time(t[2])) / n
    ms = max_over_ranks(ms, world, dev)
    del g, fl
    total = sum_over_ranks(bytes_step, world, dev)
    return {"value": round(total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ms, 4),
            "how": "one step (two L2 flushes included) captured in a CUDA graph and replayed; "
                   "the flushes' own replay time subtracted"}


def run_e2e(path, args, stream, reuse, world, dev, bytes_step):
    """Host buffers in, host result out, through the same C-ABI calls.

    Every step copies its inputs (x, topk_idx, topk_weights) from pinned host
    memory and its output back to pinned host memory.  Steps are independent,
    so they are pipelined over two buffer slots: uploads on one stream,
    kernels on the bench's stream, downloads on a third, ordered by events --
    the kernels of step i overlap the upload of step i+1 and the download of
    step i-1, and the two PCIe directions run at the same time."""
    import torch
    wl = path.wl
    x_h = wl.x.pin_memory()
    idx_h = wl.topk_idx.pin_memory()
    w_h = wl.topk_weights.pin_memory()
    out_h = [torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_d = [torch.empty_like(path.x) for _ in range(2)]
    idx_d = [torch.empty_like(path.idx) for _ in range(2)]
    w_d = [torch.empty_like(path.w) for _ in range(2)]
    out_d = [torch.empty_like(path.out) for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in_ready", "in_free", "out_ready", "out_free")}
    sptr = stream.cuda_stream
    n = max(4, min(args.steps, 20))

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(ev["in_free"][b])
            x_d[b].copy_(x_h, non_blocking=True)
            idx_d[b].copy_(idx_h, non_blocking=True)
            w_d[b].copy_(w_h, non_blocking=True)
            ev["in_ready"][b].record(up)
        stream.wait_event(ev["in_ready"][b])
        if i >= 2:
            stream.wait_event(ev["out_free"][b])
        path.layout(sptr, idx=idx_d[b], w=w_d[b])
        for _ in range(reuse):
            path.dispatch(sptr, x=x_d[b], idx=idx_d[b])
            path.combine(sptr, out=out_d[b], w=w_d[b])
        ev["in_free"][b].record(stream)
        ev["out_ready"][b].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev["out_ready"][b])
            out_h[b].copy_(out_d[b], non_blocking=True)
            ev["out_free"][b].record(down)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    t0.record(up)
    for i in range(n):
        e2e_step(i)
    t1.record(down)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / n
    ms = max_over_ranks(ms, world, dev)
    total = sum_over_ranks(bytes_step, world, dev)
    h2d = x_h.numel() * 2 + idx_h.numel() * 8 + w_h.numel() * 4
    d2h = out_h[0].numel() * 2

    # the PCIe floor of a pipelined step: one step's uploads and its download
    # issued together on the two copy streams, no kernels
    def copies_ms(do_up, do_down, reps=5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(up)
        down.wait_event(a)
        for _ in range(reps):
            if do_up:
                with torch.cuda.stream(up):
                    x_d[0].copy_(x_h, non_blocking=True)
                    idx_d[0].copy_(idx_h, non_blocking=True)
                    w_d[0].copy_(w_h, non_blocking=True)
            if do_down:
                with torch.cuda.stream(down):
                    out_h[1].copy_(out_d[1], non_blocking=True)
        up.wait_stream(down)
        b.record(up)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    h2d_ms, d2h_ms, both_ms = copies_ms(True, False), copies_ms(False, True), copies_ms(True, True)
    floor_ms = max_over_ranks(both_ms, world, dev)
    return {"value": round(total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelining": "two buffer slots; uploads, kernels and downloads on three streams",
            "pcie": {"h2d_gbs_alone": round(h2d / (h2d_ms * 1e-3) / 1e9, 1),
                     "d2h_gbs_alone": round(d2h / (d2h_ms * 1e-3) / 1e9, 1),
                     "floor_ms_per_step": round(floor_ms, 4),
                     "frac": round(floor_ms / ms, 4),
                     "note": "floor = one step's uploads and download issued together, no kernels"}}


# ----------------------------------------------------------------------------
# Expert GEMM with the fused combine (ep_expert_combine)
# ----------------------------------------------------------------------------
EGEMM = dict(T=4096, H=7168, E=32, R=8, K=8, A=128, router="topk", seed=5, I=2048)
EGEMM_DESC = ("one expert-parallel rank of a DeepSeek-V3 layer: 32 local experts receiving 4096 tokens x "
              "top-8 (32768 rows, 1024 per expert, align 128); expert down projection 2048 -> 7168 bf16 "
              "with the top-k weighted combine in the epilogue")
EGEMM_DESC_FP8 = EGEMM_DESC.replace("2048 -> 7168 bf16", "2048 -> 7168 E4M3 (1x128 row scales, 128x128 "
                                     "expert-matrix scales)")


def run_peer(args, world, rank, local):
    """ep_dispatch_peer + ep_combine_peer on the named workload, its R
    destination buffers all on this GPU (the addressing and store pattern of
    the cross-GPU exchange, at this GPU's own bandwidth), timed beside
    ep_dispatch + ep_combine on the same layout.  Layout is computed once,
    outside the timed region."""
    import numpy as np
    import torch

    import combine_ep_get_08_b200 as ep
    import workloads

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    from combine_ep_get_08_b200 import build_lib
    if rank == 0:
        build_lib.build()
    barrier(world)
    base = workloads.CONFIGS[args.config]
    fp8 = base["fp8"]
    wl = workloads.generate(None, seed=base["seed"] + 1000 * rank,
                            **{k: v for k, v in base.items() if k not in ("reuse", "seed")})
    cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A)
    h = ep.ep_handle_create(cfg)
    if args.sm_limit:
        ep.ep_set_sm_limit(h, args.sm_limit)
    x, idx, tw = wl.x.to(dev), wl.topk_idx.to(dev), wl.topk_weights.to(dev)
    roff = torch.empty(wl.R + 1, dtype=torch.int32, device=dev)
    ep.ep_get_layout(h, idx, tw, rank_offsets=roff)
    r = roff.cpu().numpy().astype(np.int64)
    rows = int(r[-1])
    seg = np.diff(r)
    # destination d holds this source's block after another source's block of
    # the same size (row0 = seg[d]): non-zero offsets, 2x the rows in memory
    row0 = seg.astype(np.int32)
    n_d = [int(2 * seg[d]) + 1 for d in range(wl.R)]
    ybufs = [torch.empty((n, wl.H), dtype=torch.bfloat16, device=dev) for n in n_d]
    y_bases = torch.tensor([b.data_ptr() for b in ybufs], dtype=torch.int64, device=dev)
    row0_d = torch.from_numpy(row0).to(dev)
    cap = max(ep.ep_capacity_rows(cfg), 1)
    y_local = torch.empty((cap, wl.H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
    flush = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    cs = stream.cuda_stream
    if fp8:
        qbufs = [torch.empty((n, wl.H), dtype=torch.uint8, device=dev) for n in n_d]
        sbufs = [torch.empty((n, wl.H // 128), dtype=torch.float32, device=dev) for n in n_d]
        q_bases = torch.tensor([b.data_ptr() for b in qbufs], dtype=torch.int64, device=dev)
        s_bases = torch.tensor([b.data_ptr() for b in sbufs], dtype=torch.int64, device=dev)
        recv_q = torch.empty((cap, wl.H), dtype=torch.uint8, device=dev)
        recv_s = torch.empty((cap, wl.H // 128), dtype=torch.float32, device=dev)
        d_peer = lambda: ep.ep_dispatch_peer_fp8(h, x, q_bases, s_bases, row0_d, stream=cs)  # noqa: E731
        d_local = lambda: ep.ep_dispatch_fp8(h, x, recv_q, recv_s, stream=cs)  # noqa: E731
    else:
        rbufs = [torch.empty((n, wl.H), dtype=torch.bfloat16, device=dev) for n in n_d]
        r_bases = torch.tensor([b.data_ptr() for b in rbufs], dtype=torch.int64, device=dev)
        recv = torch.empty((cap, wl.H), dtype=torch.bfloat16, device=dev)
        d_peer = lambda: ep.ep_dispatch_peer(h, x, r_bases, row0_d, stream=cs)  # noqa: E731
        d_local = lambda: ep.ep_dispatch(h, x, recv, stream=cs)  # noqa: E731
    calls = {
        "dispatch_peer": d_peer,
        "combine_peer": lambda: ep.ep_combine_peer(h, y_bases, row0_d, tw, out, stream=cs),
        "dispatch": d_local,
        "combine": lambda: ep.ep_combine(h, y_local, tw, out, stream=cs),
    }
    for _ in range(args.warmup):
        for f in calls.values():
            f()
    torch.cuda.synchronize()
    ms = {k: [] for k in calls}
    launches0 = ep.ep_launch_count()
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        for _ in range(args.steps):
            for k, f in calls.items():
                flush.sum()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                f()
                e1.record(stream)
                ms[k].append((e0, e1))
        torch.cuda.synchronize()
    barrier(world)
    launches = ep.ep_launch_count() - launches0
    us = {k: statistics.mean(a.elapsed_time(b) for a, b in v) * 1e3 for k, v in ms.items()}
    b_dis = dispatch_bytes(wl.T, wl.H, wl.K, rows, fp8)
    b_com = combine_bytes(wl.T, wl.H, wl.K)
    peer_ms = sum(a.elapsed_time(b) for k in ("dispatch_peer", "combine_peer") for a, b in ms[k])
    total_ms = max_over_ranks(peer_ms, world, dev)
    all_bytes = sum_over_ranks((b_dis + b_com) * args.steps, world, dev)
    peak, peak_src = measured_peak()
    dom = "dispatch_peer" if us["dispatch_peer"] >= us["combine_peer"] else "combine_peer"
    dom_bytes = b_dis if dom == "dispatch_peer" else b_com
    status = ep.ep_get_status(h)
    ep.ep_handle_destroy(h)
    if rank == 0:
        achieved = dom_bytes / (us[dom] * 1e-6) / 1e9
        line = {
            "metric": "peer dispatch + combine algorithmic GB/s", "unit": "GB/s",
            "value": round(all_bytes / (total_ms * 1e-3) / 1e9, 1),
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3+bf16" if fp8 else "bf16", "data": "synthetic",
            "config": {"workload": workloads.DESCRIPTIONS[args.config], "name": args.config,
                       "destinations": wl.R, "placement": "all destination buffers on this GPU",
                       "rows": rows, "l2": "flushed (256 MiB read, outside the timed events) before each call"},
            "kernels_us": {k: round(v, 2) for k, v in us.items()},
            "peer_vs_local": {"dispatch": round(us["dispatch"] / us["dispatch_peer"], 3),
                              "combine": round(us["combine"] / us["combine_peer"], 3)},
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                         "peak_source": peak_src, "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": None},
            "gpu_launches": int(launches), "clocks": sampler.summary(), "device_status": int(status),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def expert_gemm_inputs(dev, fp8: bool, rank: int = 0):
    """Handle, layout and synthetic operands of the expert GEMM workload (EGEMM).
    bf16: act ~ N(0,1), W_e ~ N(0,1)/sqrt(I).  E4M3: codes of 32*N(0,1) (saturating
    cast), row scales U(1/64, 1/16) per 128 columns, expert scales
    U(0.5, 1.5)/(32*sqrt(I)) per 128 x 128 block."""
    import torch

    import combine_ep_get_08_b200 as ep
    import workloads

    c = dict(EGEMM)
    I = c.pop("I")
    seed = c.pop("seed") + 1000 * rank
    wl = workloads.generate(None, seed=seed, with_x=False, **c)
    N = wl.H
    cfg = ep.make_config(wl.T, wl.H, wl.E, wl.R, wl.K, wl.A)
    h = ep.ep_handle_create(cfg)
    idx, tw = wl.topk_idx.to(dev), wl.topk_weights.to(dev)
    ep.ep_get_layout(h, idx, tw)
    rows = ep.ep_get_num_rows(h)
    cap = ep.ep_capacity_rows(cfg)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    ops = {"wl": wl, "h": h, "I": I, "N": N, "rows": rows, "cap": cap, "tw": tw, "fp8": fp8,
           "acc": torch.empty((wl.T, N), dtype=torch.float32, device=dev),
           "out": torch.empty((wl.T, N), dtype=torch.bfloat16, device=dev)}
    if fp8:
        def e4m3(shape):
            v = torch.randn(shape, generator=gen, device=dev) * 32.0
            return v.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
        ops["act"] = e4m3((cap, I))
        ops["sa"] = torch.rand((cap, I // 128), generator=gen, device=dev) * (3.0 / 64.0) + 1.0 / 64.0
        ops["w"] = e4m3((wl.E, N, I))
        ops["sw"] = (torch.rand((wl.E, N // 128, I // 128), generator=gen, device=dev) + 0.5) / (32.0 * I ** 0.5)
    else:
        ops["act"] = torch.randn((cap, I), generator=gen, device=dev).to(torch.bfloat16)
        ops["w"] = (torch.randn((wl.E, N, I), generator=gen, device=dev) / I ** 0.5).to(torch.bfloat16)
    return ops


def expert_gemm_call(o, stream):
    import combine_ep_get_08_b200 as ep
    if o["fp8"]:
        ep.ep_expert_combine_fp8(o["h"], o["act"], o["sa"], o["I"], o["w"], o["sw"], o["N"], o["tw"], o["acc"],
                                 o["out"], stream=stream.cuda_stream)
    else:
        ep.ep_expert_combine(o["h"], o["act"], o["I"], o["w"], o["N"], o["tw"], o["acc"], o["out"],
                             stream=stream.cuda_stream)


def gemm_peak(fp8: bool):
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16 = float(json.load(f)["bf16_tflops"])
        src = "measured burst (MEASURED_PEAKS.json bf16_tflops)"
    except Exception:  # noqa: BLE001
        bf16, src = 1590.0, "fallback 1.59 PFLOP/s"
    if fp8:
        return 2.0 * bf16, src + " x 2 (nominal dense FP8 / bf16 ratio, 4.5 / 2.25 PFLOP/s)"
    return bf16, src


def time_expert_gemm(o, steps, warmup, flush, stream):
    """Per-call CUDA-event times (ms) of the expert GEMM, L2 flushed before each call."""
    import torch
    for _ in range(warmup):
        expert_gemm_call(o, stream)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in evs:
        flush.sum()
        e0.record(stream)
        expert_gemm_call(o, stream)
        e1.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def expert_gemm_summary(o, ms):
    """Per-config entry of the default bench line for one expert GEMM dtype."""
    wl = o["wl"]
    pairs = int((wl.topk_idx >= 0).sum())
    flops_call = 2.0 * pairs * o["N"] * o["I"]
    peak, src = gemm_peak(o["fp8"])
    mean_ms = statistics.mean(ms)
    tf = flops_call / (mean_ms * 1e-3) / 1e12
    return {"workload": EGEMM_DESC if not o["fp8"] else EGEMM_DESC_FP8, "steps": len(ms),
            "us_per_call": round(mean_ms * 1e3, 2), "tflops": round(tf, 1), "peak": peak, "peak_source": src,
            "frac": round(tf / peak, 4), "dtype": "e4m3" if o["fp8"] else "bf16"}


def run_expert_gemm(args, world, rank, local):
    import numpy as np
    import torch

    import combine_ep_get_08_b200 as ep
    import workloads

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    from combine_ep_get_08_b200 import build_lib
    if rank == 0:
        build_lib.build()
    barrier(world)
    fp8 = args.gemm_dtype == "e4m3"
    o = expert_gemm_inputs(dev, fp8, rank)
    wl, h, I, N, rows = o["wl"], o["h"], o["I"], o["N"], o["rows"]
    if args.sm_limit:
        ep.ep_set_sm_limit(h, args.sm_limit)
    flush = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        expert_gemm_call(o, stream)
    torch.cuda.synchronize()
    launches0 = ep.ep_launch_count()
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        ms = time_expert_gemm(o, args.steps, 0, flush, stream)
    barrier(world)
    launches = ep.ep_launch_count() - launches0
    total_ms = max_over_ranks(sum(ms), world, dev)
    pairs = int((wl.topk_idx >= 0).sum())
    flops_call = 2.0 * pairs * N * I               # algorithmic: real rows only
    all_flops = sum_over_ranks(flops_call * args.steps, world, dev)
    tflops = all_flops / (total_ms * 1e-3) / 1e12
    status = ep.ep_get_status(h)
    peak, peak_src = gemm_peak(fp8)
    mean_ms = statistics.mean(ms)
    kernel = "gemm_combine_fp8_kernel" if fp8 else "gemm_combine_kernel"
    if rank == 0:
        line = {
            "metric": ("expert GEMM (E4M3) + fused combine TFLOP/s" if fp8
                       else "expert GEMM + fused combine TFLOP/s"),
            "value": round(tflops, 1), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic",
            "config": {"workload": EGEMM_DESC_FP8 if fp8 else EGEMM_DESC, "rows": rows,
                       "padded_rows_computed": rows, "pairs": pairs,
                       "inner": I, "n_out": N, "sm_limit": args.sm_limit or None,
                       "l2": "flushed (256 MiB read, outside the timed events) before each call"},
            "roofline": {"bound": "tensor", "kernel": kernel + " (+ memset and bf16 rounding)",
                         "achieved": round(flops_call / (mean_ms * 1e-3) / 1e12, 1), "peak": peak,
                         "peak_source": peak_src, "unit": "TFLOP/s",
                         "frac": round(flops_call / (mean_ms * 1e-3) / 1e12 / peak, 4), "traffic": None},
            "gpu_launches": int(launches), "clocks": sampler.summary(), "device_status": int(status),
        }
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            oracle.build()
            ol = oracle.layout(wl.topk_idx.numpy(), wl.E, wl.R, wl.A)
            if fp8:
                a_h, sa_h = o["act"][:rows].cpu().numpy(), o["sa"][:rows].cpu().numpy()
                w_h, sw_h = o["w"].cpu().numpy(), o["sw"].cpu().numpy()
                one = lambda t: oracle.expert_combine_fp8(  # noqa: E731
                    a_h, sa_h, w_h, sw_h, wl.topk_idx.numpy(), ol.pos, wl.topk_weights.numpy(),
                    sel_tokens=np.array([t], np.int32))
            else:
                act_b = workloads.bf16_bits(o["act"][:rows])
                w_b = workloads.bf16_bits(o["w"])
                one = lambda t: oracle.expert_combine(  # noqa: E731
                    act_b, w_b, wl.topk_idx.numpy(), ol.pos, wl.topk_weights.numpy(), np.array([t], np.int32))
            n_tok, t0 = 0, time.perf_counter()
            while time.perf_counter() - t0 < args.cpu_budget:
                one(n_tok % wl.T)
                n_tok += 1
            el = time.perf_counter() - t0
            line["cpu_baseline"] = {
                "value": round(2.0 * wl.K * N * I * n_tok / el / 1e12, 6), "unit": "TFLOP/s", "cores": 1,
                "kind": "oracle", "sample": f"{n_tok} token(s) of the same workload ({el:.1f} s, single thread, fp64)",
                "host": host_cpu()}
        print(json.dumps(line), flush=True)
    ep.ep_handle_destroy(h)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def ncu_ingest(rep: str, workload: str) -> int:
    """Record DRAM bytes per launch of the layout / dispatch / combine kernels
    from an ncu report (``ncu -i REP --page raw --csv``; per kernel the mean
    over its captured launches) into profiles/ncu_traffic.json under
    `workload`, stamped with the digest of the current kernel sources.
    Entries taken on other sources are dropped."""
    import csv
    import io
    import subprocess

    raw = subprocess.run(["ncu", "-i", rep, "--page", "raw", "--csv"], check=True,
                         capture_output=True, text=True).stdout
    rows = list(csv.reader(io.StringIO(raw)))
    hdr = rows[0]
    col = {k: hdr.index(k) for k in ("Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum")}
    unit = rows[1]
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    per_role = {}
    for r in rows[2:]:
        name = r[col["Kernel Name"]]
        # a kernel that dispatches (the layout fused in or not) is the dispatch
        role = ("dispatch" if "dispatch" in name else "layout" if "layout" in name
                else "combine" if "combine" in name else None)
        if role is None:
            continue
        rd = float(r[col["dram__bytes_read.sum"]].replace(",", "")) * scale[unit[col["dram__bytes_read.sum"]]]
        wr = float(r[col["dram__bytes_write.sum"]].replace(",", "")) * scale[unit[col["dram__bytes_write.sum"]]]
        short = name.split("(")[0].replace("void ", "").split("::")[-1]
        per_role.setdefault(role, {"kernel": short, "n": 0, "rd": 0.0, "wr": 0.0})
        e = per_role[role]
        e["n"] += 1
        e["rd"] += rd
        e["wr"] += wr
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    digest = kernel_source_digest()
    try:
        with open(path) as f:
            data = json.load(f)
    except Exception:  # noqa: BLE001
        data = {}
    if data.get("source_digest") != digest:
        data = {"source_digest": digest, "roles": {}}
    data["how"] = ("one capture per kernel: ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum "
                   "--clock-control none -k <kernel> -s <warm-up launches> -c 1 on the bench command; "
                   "caches are flushed between replays; each capture's roles are merged into its workload")
    data.setdefault("roles", {}).setdefault(workload, {}).update({
        role: {"kernel": e["kernel"], "launches": e["n"], "dram_bytes_read": round(e["rd"] / e["n"]),
               "dram_bytes_write": round(e["wr"] / e["n"]),
               "dram_bytes_per_launch": round((e["rd"] + e["wr"]) / e["n"])}
        for role, e in per_role.items()})
    with open(path, "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")
    print(json.dumps(data["roles"][workload], indent=1))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--config", default="dsv3", choices=["tiny", "dsv3", "decode", "skew", "large"])
    ap.add_argument("--reuse", type=int, default=None, help="dispatch+combine calls per layout")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds for the oracle baseline")
    ap.add_argument("--ref-tokens", type=int, default=4096, help="tokens per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per_config block (the other four workloads, measured after dsv3)")
    ap.add_argument("--sm-limit", type=int, default=0, help="SMs dispatch/combine may occupy (0: all)")
    ap.add_argument("--mode", choices=["normal", "ll", "fused"], default="normal",
                    help="layout: normal (padded, ep_get_layout then ep_dispatch), fused (ep_layout_dispatch) "
                         "or low-latency static slots (ep_ll_*)")
    ap.add_argument("--ll-slots", type=int, default=0, help="slots per expert in --mode ll (0: T)")
    ap.add_argument("--ncu-ingest", metavar="REP", help="record DRAM traffic from an ncu report and exit")
    ap.add_argument("--peer", action="store_true",
                    help="time ep_dispatch_peer + ep_combine_peer (R destination buffers on this GPU)")
    ap.add_argument("--gemm-dtype", choices=["bf16", "e4m3"], default="bf16",
                    help="operand type of --expert-gemm")
    ap.add_argument("--expert-gemm", action="store_true",
                    help="time ep_expert_combine (expert GEMM + fused combine) instead of the step")
    args = ap.parse_args(argv)
    if args.ncu_ingest:
        return ncu_ingest(args.ncu_ingest, args.config + ("" if args.mode == "normal" else "-" + args.mode))
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 must be launched with torchrun (one process per GPU)")
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.expert_gemm:
        return run_expert_gemm(args, world, rank, local)
    if args.peer:
        return run_peer(args, world, rank, local)
    return run_cuda(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
