"""Expert parallelism across GPUs: the exchange step (one process per GPU).

With W ranks in a torch.distributed group, rank g owns experts
[g*L, (g+1)*L), L = E / W (the even split of "blog.hotdry.top ...
deepep-expert-parallel-alltoall", buffer section: num_experts % group.size()
== 0).  Each rank routes its own T tokens:

  1. ep_get_layout with num_ranks = W: the received-row layout is expert-major,
     so the rows bound for rank r form one contiguous segment
     [rank_offsets[r], rank_offsets[r+1]) (padded per expert to
     expert_alignment);
  2. ep_dispatch / ep_dispatch_fp8 writes those rows (the send buffer);
  3. exchange_rows sends segment r to rank r with one all_to_all (NCCL over
     NVLink between the GPUs of a node);
  4. the experts run on the received rows;
  5. return_rows sends every expert output row back to its source rank, into
     the row it was sent from, and ep_combine reduces them there.

This is the normal-mode dispatch / combine golden path of DeepEP
("bowenzhou.top/repos/deepep/01-overview" section 1.3: dispatch, experts,
combine(x, handle)).  The row counts are exchanged first and read on the
host (all_to_all takes host split sizes) -- the do_cpu_sync of section 1.1.
Received rows are grouped by source rank; inside each source's block, by
local expert, each segment padded to expert_alignment (``ExchangePlan``
gives the sizes).

The functions take tensors on the group's device (CUDA with NCCL, CPU with
gloo) and hold no arithmetic of their own: the rows are the dispatch
kernel's output and the reduction is ep_combine.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass
class ExchangePlan:
    world: int
    local_experts: int                 # L = E / W
    send_rows: list                    # rows to each destination rank (padded segments)
    recv_rows: list                    # rows from each source rank
    recv_expert_pairs: torch.Tensor    # [W, L] int64 (host): pairs of local expert l from source s
    recv_expert_rows: torch.Tensor     # [W, L] int64 (host): the same padded to expert_alignment

    @property
    def total_send(self) -> int:
        return int(sum(self.send_rows))

    @property
    def total_recv(self) -> int:
        return int(sum(self.recv_rows))


def plan_exchange(num_tokens_per_expert, expert_alignment: int, group=None, device=None) -> ExchangePlan:
    """Row counts of the exchange from this rank's per-expert pair counts.

    num_tokens_per_expert: E counts of this rank's layout (any device).  One
    all_to_all of the counts (each rank sends the L counts of rank r's
    experts to rank r); everything else is host arithmetic on them."""
    import torch.distributed as dist

    W = dist.get_world_size(group)
    cnt = torch.as_tensor(num_tokens_per_expert).to(torch.int64).cpu()
    E = cnt.numel()
    if E % W != 0:
        raise ValueError(f"num_experts {E} is not a multiple of the group size {W}")
    L = E // W
    A = int(expert_alignment)
    padded = (cnt + A - 1) // A * A
    send_rows = padded.view(W, L).sum(1).tolist()
    dev = torch.device("cpu") if device is None else torch.device(device)
    send_cnt = cnt.view(W, L).contiguous().to(dev)
    recv_cnt = torch.empty_like(send_cnt)
    dist.all_to_all_single(recv_cnt, send_cnt, group=group)
    recv_cnt = recv_cnt.cpu()
    recv_padded = (recv_cnt + A - 1) // A * A
    return ExchangePlan(world=W, local_experts=L, send_rows=[int(v) for v in send_rows],
                        recv_rows=[int(v) for v in recv_padded.sum(1).tolist()],
                        recv_expert_pairs=recv_cnt, recv_expert_rows=recv_padded)


def exchange_rows(send: torch.Tensor, plan: ExchangePlan, group=None) -> torch.Tensor:
    """Send rows [rank_offsets[r], rank_offsets[r+1]) of `send` to rank r;
    returns the received rows, grouped by source rank."""
    import torch.distributed as dist

    out = torch.empty((plan.total_recv,) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
    dist.all_to_all_single(out, send[:plan.total_send].contiguous(), output_split_sizes=plan.recv_rows,
                           input_split_sizes=plan.send_rows, group=group)
    return out


def return_rows(y_recv: torch.Tensor, plan: ExchangePlan, out: torch.Tensor | None = None,
                group=None) -> torch.Tensor:
    """The reverse exchange: row i of each source's block goes back to row
    rank_offsets[r] + i of that source.  `out` (optional) must hold at least
    plan.total_send rows; rows past them are left as they are."""
    import torch.distributed as dist

    if out is None:
        out = torch.empty((plan.total_send,) + tuple(y_recv.shape[1:]), dtype=y_recv.dtype, device=y_recv.device)
    dst = out[:plan.total_send]
    if dst.is_contiguous():
        dist.all_to_all_single(dst, y_recv[:plan.total_recv].contiguous(), output_split_sizes=plan.send_rows,
                               input_split_sizes=plan.recv_rows, group=group)
    else:
        tmp = torch.empty_like(dst)
        dist.all_to_all_single(tmp, y_recv[:plan.total_recv].contiguous(), output_split_sizes=plan.send_rows,
                               input_split_sizes=plan.recv_rows, group=group)
        dst.copy_(tmp)
    return out


def dispatch(h: int, x: torch.Tensor, topk_idx: torch.Tensor, topk_weights, send: torch.Tensor, cfg,
             group=None, stream=None):
    """Layout, dispatch and exchange on this rank's GPU (bf16 rows).

    cfg.num_ranks must equal the group size.  `send` is the [capacity, H]
    bf16 send buffer.  Returns (received rows, plan)."""
    import torch.distributed as dist

    from . import ep_dispatch, ep_get_layout

    if cfg.num_ranks != dist.get_world_size(group):
        raise ValueError("cfg.num_ranks must equal the process group's size")
    cnt = torch.empty((cfg.num_experts,), dtype=torch.int32, device=x.device)
    ep_get_layout(h, topk_idx, topk_weights, cnt, stream=stream)
    ep_dispatch(h, x, send, stream=stream)
    plan = plan_exchange(cnt, cfg.expert_alignment, group=group, device=x.device)
    return exchange_rows(send, plan, group=group), plan


def combine(h: int, y_recv: torch.Tensor, plan: ExchangePlan, topk_weights: torch.Tensor, out: torch.Tensor,
            y_send: torch.Tensor, group=None, stream=None) -> torch.Tensor:
    """Reverse exchange of the expert outputs into `y_send` ([capacity, H]
    bf16), then ep_combine on this rank."""
    from . import ep_combine

    return_rows(y_recv, plan, out=y_send, group=group)
    ep_combine(h, y_send, topk_weights, out, stream=stream)
    return out
