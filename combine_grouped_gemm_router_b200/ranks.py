"""The MoE layer over W real ranks, one process per GPU.

The dataflow of "MoE 专家并行的 All-to-All 通信瓶颈", §All-to-All 分发与回收的机制 (its flowchart):
route Top-K, pack by destination card, all-to-all, group by expert, grouped GEMM, pack by
source, all-to-all, weighted merge into the original token order. Rank r holds the tokens of
home shard r and experts [r E/W, (r+1) E/W):

1. route its own tokens (``moe_route``);
2. all-gather every rank's top-K (N*K int32: small), so that every rank runs the whole batch's
   bookkeeping and the W ranks keep exactly the assignments one dispatch of the whole batch
   keeps (capacity is per expert over all ranks' tokens, in the same priority order);
3. ``moe_dispatch_rank``: the bookkeeping, and this rank's rows packed by destination rank;
4. the exchange (``exchange.exchange_rows``: an all-to-allv sized by the traffic matrix D);
5. ``moe_regroup_rows`` (direction 0): the received rows into this rank's experts' order;
6. ``moe_expert_gemm`` over this rank's experts;
7. ``moe_regroup_rows`` (direction 1): the expert outputs back into the received order;
8. the return exchange (the same all-to-allv with the splits swapped);
9. ``moe_combine`` with each slot's row in the returned buffer (``send_row_of``).

Every step that touches rows runs in the library's kernels; this module orchestrates them
and the collectives (the host reads only D, W*W integers, to size the exchanges). The kernels
are reached through an ``ops`` object so that the orchestration can also run on CPU ranks
with any implementation of the same contracts; ``CudaOps`` is the library's.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (MOE_FLAG_H_BF16, MoeShape, make_shape, moe_combine, moe_dispatch_rank,
               moe_expert_gemm, moe_regroup_rows, moe_route, moe_rows_alloc, moe_workspace_size)
from .exchange import exchange_rows


class CudaOps:
    """The library's kernels on device tensors (the current CUDA stream)."""

    def __init__(self):
        self._m = dict(make_shape=make_shape, moe_combine=moe_combine,
                       moe_dispatch_rank=moe_dispatch_rank, moe_expert_gemm=moe_expert_gemm,
                       moe_regroup_rows=moe_regroup_rows, moe_route=moe_route,
                       moe_rows_alloc=moe_rows_alloc, moe_workspace_size=moe_workspace_size)
        self.MoeShape = MoeShape

    def route(self, shape_local, x, w_router, bias):
        m = self._m
        N, K = shape_local.N, shape_local.K
        topk = torch.empty(N, K, dtype=torch.int32, device=x.device)
        topw = torch.empty(N, K, dtype=torch.float32, device=x.device)
        ws = torch.empty(max(m["moe_workspace_size"](shape_local), 256), dtype=torch.uint8,
                         device=x.device)
        m["moe_route"](shape_local, x, w_router, bias, topk, topw, None, ws)
        return topk, topw

    def dispatch_rank(self, shape, rank, x_local, topk_all):
        m = self._m
        dev = x_local.device
        N, E, K, W, d = shape.N, shape.E, shape.K, shape.W, shape.d
        RA = m["moe_rows_alloc"](shape)
        i32 = dict(dtype=torch.int32, device=dev)
        b = dict(counts=torch.empty(E, **i32), kept=torch.empty(E, **i32),
                 offsets=torch.empty(E + 1, **i32), row_of=torch.empty(N * K, **i32),
                 assign=torch.empty(RA, **i32), packed_row_of=torch.empty(N * K, **i32),
                 send_row_of=torch.empty((N // W) * K, **i32),
                 x_send=torch.empty(RA, d, dtype=torch.bfloat16, device=dev),
                 D=torch.empty(W * W, dtype=torch.int64, device=dev),
                 pk_off=torch.empty(W * W + 1, dtype=torch.int64, device=dev))
        ws = torch.empty(m["moe_workspace_size"](shape), dtype=torch.uint8, device=dev)
        m["moe_dispatch_rank"](shape, rank, x_local, topk_all, b["counts"], b["kept"],
                               b["offsets"], b["row_of"], b["assign"], b["packed_row_of"],
                               b["send_row_of"], b["x_send"], b["D"], b["pk_off"], ws=ws)
        return b

    def regroup(self, shape, rank, direction, src, book, rows):
        m = self._m
        W, E = shape.W, shape.E
        dst = src.new_empty((rows + 128,) + tuple(src.shape[1:])) if direction == 0 else \
            src.new_empty((rows,) + tuple(src.shape[1:]))
        off_local = torch.empty(E // W + 1, dtype=torch.int32, device=src.device)
        m["moe_regroup_rows"](shape, rank, direction, src, dst, book["assign"],
                              book["packed_row_of"], book["offsets"], book["pk_off"],
                              off_local)
        return dst, off_local

    def experts(self, shape, rank, x_sorted, offsets_local, rows, w1, w3, w2):
        """This rank's experts over its sorted rows: fp32 y [rows (+128)][d]."""
        m = self._m
        El = shape.E // shape.W
        gshape = m["make_shape"](rows, shape.d, shape.f, El, 1, 1, 0.0,
                                 h_bf16=bool(shape.flags & MOE_FLAG_H_BF16))
        y = torch.empty(rows + 128, shape.d, dtype=torch.float32, device=x_sorted.device)
        h = torch.empty(rows + 128, shape.f,
                        dtype=torch.bfloat16 if shape.flags & MOE_FLAG_H_BF16 else torch.float16,
                        device=x_sorted.device)
        m["moe_expert_gemm"](gshape, x_sorted, offsets_local, w1, w3, w2, h, y)
        return y

    def combine(self, shape_local, y, row_of, topk_w, residual, out):
        self._m["moe_combine"](shape_local, y, row_of, topk_w, out, residual=residual)
        return out


def layer_ranks(shape, x_local, w_router, bias, w1_local, w3_local, w2_local, out,
                residual=None, group=None, ops=None) -> dict:
    """The layer of rank ``dist.get_rank(group)`` of W ranks. shape: the whole batch (N tokens
    over W ranks = the group's size). x_local [N/W][d]: this rank's tokens; w_router, bias: the
    router (the same on every rank); w1_local, w3_local [E/W][f][d], w2_local [E/W][d][f]: this
    rank's experts (W2 as the fp16 copy unless the shape asks for bf16 h); out [N/W][d]: the
    layer output of this rank's tokens (fp32, or bf16 with the out_bf16 flag); residual
    (nullable) as for moe_combine. Returns the bookkeeping (the whole batch's, identical on
    every rank) and this rank's routing."""
    ops = ops or CudaOps()
    W = dist.get_world_size(group)
    r = dist.get_rank(group)
    if shape.W != W or shape.N % W or shape.E % W:
        raise ValueError("shape.W must be the group's size, with N and E divisible by it")
    local = _local_shape(shape, ops)
    topk, topw = ops.route(local, x_local, w_router, bias)
    parts = [torch.empty_like(topk) for _ in range(W)]
    dist.all_gather(parts, topk.contiguous(), group=group)
    topk_all = torch.cat(parts, 0)
    book = ops.dispatch_rank(shape, r, x_local, topk_all)
    D = book["D"].cpu().reshape(W, W)
    send_rows = int(D[r].sum())
    recv = exchange_rows(book["x_send"][:send_rows], D, group)
    rows = recv.shape[0]
    x_sorted, off_local = ops.regroup(shape, r, 0, recv, book, rows)
    y = ops.experts(shape, r, x_sorted, off_local, rows, w1_local, w3_local, w2_local)
    y_back, _ = ops.regroup(shape, r, 1, y[:rows], book, rows)
    y_ret = exchange_rows(y_back, D.t().contiguous(), group)
    ops.combine(local, y_ret, book["send_row_of"], topw, residual, out)
    book.update(topk_idx=topk, topk_w=topw, topk_all=topk_all, D_host=D)
    return book


def _local_shape(shape, ops):
    """The shape of this rank's own tokens: N/W tokens, one home rank."""
    s = ops.MoeShape(shape.N // shape.W, shape.d, shape.f, shape.E, shape.K, 1,
                     shape.capacity_factor, shape.flags)
    return s
