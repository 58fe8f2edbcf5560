"""The cross-GPU exchange of combine_ep_get_08_b200.dist on CPU: world size 2
over gloo, with the rows and layouts of the oracle standing in for the
kernels (the exchange itself holds no arithmetic).

Every rank routes its own tokens over all E experts (rank g owns experts
[g*L, (g+1)*L)).  After exchange_rows, rank r must hold, for every source s
in order, exactly the rows source s laid out for rank r's experts; the count
exchange must report each (source, local expert) pair count; and
return_rows of the received rows (identity experts) must give every source
back its own rows bit for bit, so that the combine there reproduces x * sum w.
"""
import json
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

import oracle
import workloads

E, K, H, A, T = 8, 3, 32, 2, 40


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _source(s, W):
    wl = workloads.generate(None, T=T, H=H, E=E, R=W, K=K, A=A, router="topk", seed=300 + s)
    idx, w = wl.topk_idx.numpy(), wl.topk_weights.numpy()
    L = oracle.layout(idx, E, W, A, topk_weights=w)
    xb = workloads.bf16_bits(wl.x)
    rows = oracle.dispatch_bf16(xb, L.row_src)
    return wl, L, xb, rows


def _rank_main(rank, world, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    from combine_ep_get_08_b200 import dist as epd
    oracle.build()
    dist.init_process_group("gloo", rank=rank, world_size=world)
    res = {}
    try:
        wl, L, xb, rows = _source(rank, world)
        # the exchange moves rows whatever their type: carry the bf16 bits as
        # int32 pairs, a type gloo transports
        send = torch.from_numpy(np.ascontiguousarray(rows).view(np.int32).copy())
        plan = epd.plan_exchange(L.num_tokens_per_expert, A)
        recv = epd.exchange_rows(send, plan)
        # what every source laid out for this rank, in source order
        want, pairs = [], []
        Lx = E // world
        for s in range(world):
            _, Ls, _, rows_s = _source(s, world)
            a, b = Ls.rank_offsets[rank], Ls.rank_offsets[rank + 1]
            want.append(rows_s[a:b])
            pairs.append(Ls.num_tokens_per_expert[rank * Lx:(rank + 1) * Lx])
        res["forward"] = bool(np.array_equal(recv.numpy().view(np.uint16), np.concatenate(want)))
        res["pairs"] = bool(np.array_equal(plan.recv_expert_pairs.numpy(), np.array(pairs)))
        res["rows_sum"] = bool(int(plan.recv_expert_rows.sum()) == plan.total_recv)
        # identity experts: the reverse exchange returns this rank's own rows
        back = epd.return_rows(recv, plan)
        res["reverse"] = bool(np.array_equal(back.numpy().view(np.uint16), rows))
        out = oracle.combine(back.numpy().view(np.uint16), L.pos, wl.topk_weights.numpy())
        x = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        res["combine"] = bool(np.allclose(out, x * wl.topk_weights.numpy().astype(np.float64).sum(1, keepdims=True),
                                          rtol=1e-13, atol=1e-13))
        try:                                   # 7 experts cannot be split over 2 ranks
            epd.plan_exchange(torch.zeros(7, dtype=torch.int32), 1)
            res["uneven"] = False
        except ValueError:
            res["uneven"] = True
    finally:
        dist.destroy_process_group()
    with open(f"{out_path}.{rank}", "w") as f:
        json.dump(res, f)


def test_two_rank_exchange(tmp_path):
    out = str(tmp_path / "res")
    mp.spawn(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    for r in range(2):
        assert json.load(open(f"{out}.{r}")) == {"forward": True, "pairs": True, "rows_sum": True,
                                                 "reverse": True, "combine": True, "uneven": True}


def _peer_rank_main(rank, world, port, out_path):
    """peer_row0 over gloo: the blocks of all sources tile each destination's
    rows in source order, with no gap and no overlap, and placing the oracle's
    segments at those rows (what the peer dispatch does) gives exactly the
    receive buffer of the all_to_all exchange."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    from combine_ep_get_08_b200 import dist as epd
    oracle.build()
    dist.init_process_group("gloo", rank=rank, world_size=world)
    res = {}
    try:
        _, L, _, _ = _source(rank, world)
        send = np.diff(L.rank_offsets).tolist()
        row0, recv_rows = epd.peer_row0(send)
        everyone = [None] * world
        dist.all_gather_object(everyone, (send, row0, recv_rows))
        ok = True
        for r in range(world):
            at = 0
            for s in range(world):
                s_send, s_row0, _ = everyone[s]
                ok &= s_row0[r] == at                  # source s starts where s-1 ended
                at += s_send[r]
            ok &= sum(everyone[r][2]) == at            # rank r receives all of them
            ok &= everyone[r][2] == [everyone[s][0][r] for s in range(world)]
        res["tiling"] = bool(ok)
        worst = max(sum(everyone[s][0][r] for s in range(world)) for r in range(world))
        try:                                           # every rank raises the same error
            epd.peer_row0(send, max_rows=worst - 1)
            res["overflow"] = False
        except ValueError:
            res["overflow"] = True
        epd.peer_row0(send, max_rows=worst)            # exactly enough rows is fine
        # the peer placement gives the receive buffer the all_to_all gives:
        # source s's segment for this rank at row0_s[me], sources in order
        _, _, _, rows = _source(rank, world)
        plan = epd.plan_exchange(L.num_tokens_per_expert, A)
        recv = epd.exchange_rows(torch.from_numpy(np.ascontiguousarray(rows).view(np.int32).copy()), plan)
        buf = np.full((plan.total_recv, H), 0xBEEF, np.uint16)
        for s in range(world):
            _, Ls, _, rows_s = _source(s, world)
            a, b = Ls.rank_offsets[rank], Ls.rank_offsets[rank + 1]
            r0 = everyone[s][1][rank]
            buf[r0:r0 + b - a] = rows_s[a:b]
        res["same_as_all_to_all"] = bool(np.array_equal(buf, recv.numpy().view(np.uint16)))
    finally:
        dist.destroy_process_group()
    with open(f"{out_path}.{rank}", "w") as f:
        json.dump(res, f)


def test_four_rank_peer_row0(tmp_path):
    out = str(tmp_path / "peer")
    mp.spawn(_peer_rank_main, args=(4, _free_port(), out), nprocs=4, join=True)
    for r in range(4):
        assert json.load(open(f"{out}.{r}")) == {"tiling": True, "overflow": True, "same_as_all_to_all": True}
