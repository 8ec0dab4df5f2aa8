"""Exchange of packed rows between expert-parallel ranks, one process per GPU.

The single-GPU path stops at the send buffer: the dispatch packs each token row once per
destination rank, destination by destination ("MoE 专家并行的 All-to-All 通信瓶颈", §All-to-All
分发与回收的机制: pack by destination card, then the all-to-all). In a W-rank deployment rank r
sends D[r][j] rows to rank j, where D is the traffic matrix; this module moves those rows:

* ``exchange_rows``: the whole exchange as one all-to-allv collective (NCCL's over NVLink /
  NVSwitch on GPUs).
* ``exchange_rows_ordered``: the same rows moved in the order of ``moe_exchange_schedule``
  ("MoE Inference Communication", §Aurora 场景 1): phase by phase, every rank sends at most one
  piece and receives at most one piece per phase, so no receiver is fed by two senders at once,
  and the phases add up to the bound of 定理 4.2 (the busiest rank's rows).

Both take the send buffer as rows grouped by destination rank (ascending) and return the
receive buffer as rows grouped by source rank (ascending), each source's rows in the order it
sent them. Rows to oneself are copied locally. Every rank must pass the same D (``gather_traffic``
builds it from each rank's send counts). This is host-side orchestration of library
collectives; it launches no kernel of its own.
"""
from __future__ import annotations

from typing import List, Sequence

import torch
import torch.distributed as dist


def _offsets(counts: Sequence[int]) -> List[int]:
    out = [0]
    for c in counts:
        out.append(out[-1] + int(c))
    return out


def gather_traffic(send_counts: Sequence[int], group=None) -> torch.Tensor:
    """D [W][W] int64 on the host: row r = rank r's send counts (an all-gather of the rows)."""
    W = dist.get_world_size(group)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else "cpu"
    mine = torch.tensor([int(c) for c in send_counts], dtype=torch.int64, device=dev)
    if mine.numel() != W:
        raise ValueError("send_counts needs one entry per rank")
    rows = [torch.empty_like(mine) for _ in range(W)]
    dist.all_gather(rows, mine, group=group)
    return torch.stack(rows).cpu()


def exchange_rows(send: torch.Tensor, D: torch.Tensor, group=None) -> torch.Tensor:
    """All-to-allv of rows: this rank's send[rows of block j] go to rank j."""
    r = dist.get_rank(group)
    W = dist.get_world_size(group)
    D = torch.as_tensor(D, dtype=torch.int64).reshape(W, W)
    send_counts = [int(v) for v in D[r]]
    recv_counts = [int(v) for v in D[:, r]]
    if send.shape[0] != sum(send_counts):
        raise ValueError("send holds sum(D[rank]) rows")
    recv = send.new_empty((sum(recv_counts),) + tuple(send.shape[1:]))
    dist.all_to_all_single(recv, send.contiguous(), output_split_sizes=recv_counts,
                           input_split_sizes=send_counts, group=group)
    return recv


def exchange_rows_ordered(send: torch.Tensor, D: torch.Tensor, group=None,
                          schedule=None) -> torch.Tensor:
    """The exchange of ``exchange_rows`` in the contention-free order: ``schedule`` is
    (phase_dst [S][W], phase_len [S]) from moe_exchange_schedule(D) (computed here when None).
    During phase s rank i sends the next phase_len[s] rows of its block for phase_dst[s][i];
    one batch of point-to-point transfers per phase, each phase completed before the next."""
    r = dist.get_rank(group)
    W = dist.get_world_size(group)
    D = torch.as_tensor(D, dtype=torch.int64).reshape(W, W)
    if schedule is None:
        from . import moe_exchange_schedule
        dst, ln, _ = moe_exchange_schedule(D.numpy())
    else:
        dst, ln = schedule
    # every rank checks the whole schedule before any transfer, so all raise together
    total = [[0] * W for _ in range(W)]
    for s in range(len(ln)):
        busy = [int(dst[s][i]) for i in range(W) if int(dst[s][i]) >= 0]
        if len(set(busy)) != len(busy) or any(int(dst[s][i]) == i for i in range(W)) or \
                int(ln[s]) <= 0:
            raise ValueError(f"schedule phase {s} is not a matching of distinct receivers")
        for i in range(W):
            if int(dst[s][i]) >= 0:
                total[i][int(dst[s][i])] += int(ln[s])
    if any(total[i][j] != int(D[i, j]) for i in range(W) for j in range(W) if i != j):
        raise ValueError("the schedule does not deliver D")
    send_off = _offsets(D[r].tolist())
    recv_off = _offsets(D[:, r].tolist())
    if send.shape[0] != send_off[-1]:
        raise ValueError("send holds sum(D[rank]) rows")
    send = send.contiguous()
    recv = send.new_empty((recv_off[-1],) + tuple(send.shape[1:]))
    # NCCL needs every rank of the group in its first collective before point-to-point batches
    # that leave some ranks out (a phase may): a barrier makes that true whatever came before
    dist.barrier(group=group)
    # rows that stay on this rank
    recv[recv_off[r]:recv_off[r + 1]] = send[send_off[r]:send_off[r + 1]]
    sent = [0] * W  # rows of each destination block already sent
    got = [0] * W   # rows of each source block already received
    for s in range(len(ln)):
        n = int(ln[s])
        ops = []
        j = int(dst[s][r])
        if j >= 0:
            a = send_off[j] + sent[j]
            ops.append(dist.P2POp(dist.isend, send[a:a + n], j, group))
            sent[j] += n
        for i in (i for i in range(W) if int(dst[s][i]) == r):
            b = recv_off[i] + got[i]
            ops.append(dist.P2POp(dist.irecv, recv[b:b + n], i, group))
            got[i] += n
        if ops:
            for work in dist.batch_isend_irecv(ops):
                work.wait()
    return recv
