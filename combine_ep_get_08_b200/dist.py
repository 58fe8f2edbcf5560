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

dispatch_peer / combine_peer (end of the file) do the same exchange inside
the kernels: rows are stored straight into the other GPUs' buffers, mapped
with CUDA IPC, so no send buffer and no all_to_all of rows remain.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


def _join(stream) -> None:
    """The host continues once the work enqueued so far is finished.  With
    the current stream (stream None) syncing it is enough; with another
    stream the whole device is synced, since torch collectives, host reads
    and small uploads are ordered against the current stream only."""
    if stream is None:
        torch.cuda.current_stream().synchronize()
    else:
        torch.cuda.synchronize()


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
    if stream is not None:
        _join(stream)                                  # the collectives below run on the current stream
    plan = plan_exchange(cnt, cfg.expert_alignment, group=group, device=x.device)
    return exchange_rows(send, plan, group=group), plan


def combine(h: int, y_recv: torch.Tensor, plan: ExchangePlan, topk_weights: torch.Tensor, out: torch.Tensor,
            y_send: torch.Tensor, group=None, stream=None) -> torch.Tensor:
    """Reverse exchange of the expert outputs into `y_send` ([capacity, H]
    bf16), then ep_combine on this rank."""
    from . import ep_combine

    return_rows(y_recv, plan, out=y_send, group=group)
    if stream is not None:
        _join(stream)                                  # the rows came in on the current stream
    ep_combine(h, y_send, topk_weights, out, stream=stream)
    return out


# ---- the exchange inside the kernels: peer-memory dispatch / combine ----
#
# Instead of a send buffer plus all_to_all, ep_dispatch_peer stores every row
# straight into the destination GPU's receive buffer (mapped into this process
# with CUDA IPC), and ep_combine_peer reads the expert outputs back from the
# destination GPUs.  The only collectives left are on the row counts (host
# integers) and the barriers that order the ranks.


@dataclass
class PeerPlan:
    world: int
    send_rows: list      # rows this rank writes to each destination
    recv_rows: list      # rows each source writes to this rank
    row0: list           # first row of this rank's block in each destination's buffer
    row0_dev: object     # the same as a device int32 tensor (for the kernels)

    @property
    def total_recv(self) -> int:
        return int(sum(self.recv_rows))


def peer_row0(send_rows, group=None, max_rows: int | None = None):
    """Row starts of the peer exchange from every rank's send_rows.

    Sources write their blocks into a destination's buffer in rank order, so
    this rank's block in destination r starts after the rows of sources
    0..me-1 bound for r.  One all_gather of the W counts; returns
    (row0 [W], recv_rows [W]) as lists.  With max_rows, every rank checks that
    no destination receives more rows than that (the same ValueError on every
    rank, since all see the same counts)."""
    import torch.distributed as dist

    W = dist.get_world_size(group)
    me = dist.get_rank(group)
    mine = torch.as_tensor(send_rows, dtype=torch.int64).cpu().reshape(W)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    parts = [torch.empty(W, dtype=torch.int64, device=dev) for _ in range(W)]
    dist.all_gather(parts, mine.to(dev), group=group)
    S = torch.stack([p.cpu() for p in parts])          # S[s, r]: rows source s sends to rank r
    if max_rows is not None:
        worst = int(S.sum(0).max())
        if worst > max_rows:
            raise ValueError(f"a rank would receive {worst} rows, more than the buffers' {max_rows}")
    row0 = S[:me].sum(0)
    return [int(v) for v in row0.tolist()], [int(v) for v in S[:, me].tolist()]


class PeerBuffers:
    """This rank's receive buffer ([max_rows, H] bf16, or E4M3 codes
    [max_rows, H] uint8 plus fp32 scales [max_rows, H/128] with fp8=True) and
    expert-output buffer ([max_rows, H] bf16), and every rank's, mapped here
    through CUDA IPC (device address tables recv_bases, scale_bases and
    y_bases for the kernels).  Collective: every rank of the group constructs
    it with the same arguments."""

    def __init__(self, max_rows: int, hidden: int, group=None, device=None, fp8: bool = False):
        import torch.distributed as dist

        from . import ep_ipc_get_handle, ep_ipc_open_handle

        if fp8 and hidden % 128:
            raise ValueError("FP8 rows need hidden % 128 == 0")
        self.group = group
        self.fp8 = fp8
        self.max_rows = int(max_rows)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        n = max(self.max_rows, 1)
        self.recv = torch.zeros((n, hidden), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
        self.recv_scales = torch.zeros((n, hidden // 128), dtype=torch.float32, device=dev) if fp8 else None
        self.y = torch.zeros((n, hidden), dtype=torch.bfloat16, device=dev)
        local = [self.recv, self.y] + ([self.recv_scales] if fp8 else [])
        mine = [ep_ipc_get_handle(t) for t in local]
        W = dist.get_world_size(group)
        me = dist.get_rank(group)
        everyone = [None] * W
        dist.all_gather_object(everyone, mine, group=group)
        self._opened = {}                                  # handle bytes -> mapped base
        addr = [[] for _ in local]                         # per buffer kind, per rank
        for r, handles in enumerate(everyone):
            for i, (hd, off) in enumerate(handles):
                if r == me:
                    addr[i].append(local[i].data_ptr())
                    continue
                if hd not in self._opened:
                    self._opened[hd] = ep_ipc_open_handle(hd)
                addr[i].append(self._opened[hd] + off)
        table = [torch.tensor(a, dtype=torch.int64, device=dev) for a in addr]
        self.recv_bases, self.y_bases = table[0], table[1]
        self.scale_bases = table[2] if fp8 else None

    def __enter__(self) -> "PeerBuffers":
        return self

    def __exit__(self, *exc) -> None:
        self.close()

    def close(self) -> None:
        """Unmaps the other ranks' buffers (after the last kernel that uses them)."""
        from . import ep_ipc_close_handle

        torch.cuda.synchronize()
        for base in self._opened.values():
            ep_ipc_close_handle(base)
        self._opened = {}


def _fence(group, stream) -> None:
    """This rank's work so far is finished and every rank has reached here."""
    import torch.distributed as dist

    _join(stream)
    dist.barrier(group=group)


def dispatch_peer(h: int, x: torch.Tensor, topk_idx: torch.Tensor, topk_weights, cfg, bufs: PeerBuffers,
                  group=None, stream=None):
    """Layout on this GPU, then the rows go straight into the destination
    GPUs' receive buffers (E4M3 codes and scales if bufs.fp8).  Returns (the
    rows this rank received, grouped by source rank -- a view of bufs.recv,
    or (codes, scales) views with FP8 -- and the plan)."""
    import torch.distributed as dist

    from . import ep_dispatch_peer, ep_dispatch_peer_fp8, ep_get_layout

    W = dist.get_world_size(group)
    if cfg.num_ranks != W:
        raise ValueError("cfg.num_ranks must equal the process group's size")
    roff = torch.empty((W + 1,), dtype=torch.int32, device=x.device)
    ep_get_layout(h, topk_idx, topk_weights, None, None, None, None, roff, stream=stream)
    _join(stream)
    r = roff.cpu()
    send_rows = (r[1:] - r[:-1]).tolist()
    row0, recv_rows = peer_row0(send_rows, group=group, max_rows=bufs.max_rows)
    # uploaded on the current stream; the fence below finishes it before the launch
    row0_dev = torch.tensor(row0, dtype=torch.int32, device=x.device)
    plan = PeerPlan(world=W, send_rows=[int(v) for v in send_rows], recv_rows=recv_rows, row0=row0,
                    row0_dev=row0_dev)
    _fence(group, stream)                              # every destination is done with its last rows
    if bufs.fp8:
        ep_dispatch_peer_fp8(h, x, bufs.recv_bases, bufs.scale_bases, row0_dev, stream=stream)
    else:
        ep_dispatch_peer(h, x, bufs.recv_bases, row0_dev, stream=stream)
    _fence(group, stream)                              # every row has landed
    n = plan.total_recv
    if bufs.fp8:
        return (bufs.recv[:n], bufs.recv_scales[:n]), plan
    return bufs.recv[:n], plan


def combine_peer(h: int, plan: PeerPlan, topk_weights: torch.Tensor, out: torch.Tensor, bufs: PeerBuffers,
                 group=None, stream=None) -> torch.Tensor:
    """The expert outputs of this rank's received rows are in
    bufs.y[:plan.total_recv] on every rank; reads this rank's rows back from
    all of them and writes the weighted sum per token into `out`."""
    from . import ep_combine_peer

    _fence(group, stream)                              # every rank's expert outputs are complete
    ep_combine_peer(h, bufs.y_bases, plan.row0_dev, topk_weights, out, stream=stream)
    _fence(group, stream)                              # nobody overwrites y while it is read
    return out
