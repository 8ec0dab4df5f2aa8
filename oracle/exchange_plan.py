"""CPU oracle of the exchange planning: the exchange-time bound, the cost of an
expert placement and the exact optimum of the placement ILP.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` may import this module. It shares no code with the
product library.

Followed passages ("MoE Inference Communication"):

* §Aurora 场景 1, 定理 4.2: the shortest exchange of a traffic matrix D lasts
  max(largest row sum, largest column sum) of D divided by the per-GPU
  bandwidth; here in rows, without the diagonal (rows that stay on their rank
  cross no link).
* §ExFlow 形式化：整数线性规划建模: binary x[j][i][g] (expert i of layer j on
  GPU g); every GPU holds E/P experts of every layer; every expert sits on one
  GPU; a token hop from expert i of layer j to expert p of layer j+1 crosses
  GPUs (R = 1) when the two sit on different GPUs; minimise the number of
  crossing hops. The printed routing constraint names the same expert index on
  both layers, which cannot be what is meant (the hop goes from the token's
  layer-j expert to its layer-(j+1) expert); it is read as
  R[j][i][p] >= x[j][i][g] - x[j+1][p][g] and >= x[j+1][p][g] - x[j][i][g]
  for every g. Tokens with the same (i, p) hop have identical constraints, so
  the per-token R of the page are merged into one R per hop weighted by the
  hop count (the affinity counts; with K > 1 experts per token every one of the
  K x K hops of a token counts).
"""
from __future__ import annotations

import numpy as np


def exchange_bound(D) -> int:
    """max(max_i sum_{j != i} D[i][j], max_j sum_{i != j} D[i][j]) in rows."""
    off = np.array(D, dtype=np.int64, copy=True)
    np.fill_diagonal(off, 0)
    if off.size == 0:
        return 0
    return int(max(off.sum(axis=1).max(), off.sum(axis=0).max()))


def placement_cost(counts, gpu_of) -> int:
    """Hops between consecutive layers whose experts sit on different GPUs:
    sum over j, i, p of counts[j][i][p] * [gpu_of[j][i] != gpu_of[j+1][p]]."""
    counts = np.asarray(counts, dtype=np.int64)
    g = np.asarray(gpu_of)
    total = 0
    for j in range(counts.shape[0]):
        cross = g[j][:, None] != g[j + 1][None, :]
        total += int(counts[j][cross].sum())
    return total


def contiguous_placement(L: int, E: int, P: int) -> np.ndarray:
    """Expert e on GPU e // (E/P) on every layer."""
    return np.tile(np.arange(E) // (E // P), (L, 1)).astype(np.int32)


def ilp_placement(counts, P: int):
    """The page's ILP, solved exactly (scipy.optimize.milp, HiGHS branch and bound).

    counts: int64 [L-1][E][E]. Returns (optimal cost, gpu_of [L][E]).
    """
    from scipy.optimize import Bounds, LinearConstraint, milp

    counts = np.asarray(counts, dtype=np.int64)
    Lm1, E, _ = counts.shape
    L = Lm1 + 1
    share = E // P
    nx = L * E * P

    def xv(j, i, g):
        return (j * E + i) * P + g

    hops = [(j, i, p) for j in range(Lm1) for i in range(E) for p in range(E)
            if counts[j, i, p] > 0]
    nv = nx + len(hops)
    c = np.zeros(nv)
    for h, (j, i, p) in enumerate(hops):
        c[nx + h] = float(counts[j, i, p])
    rows, lo, hi = [], [], []

    def add(coefs, a, b):
        r = np.zeros(nv)
        for k, v in coefs:
            r[k] += v
        rows.append(r)
        lo.append(a)
        hi.append(b)

    for j in range(L):
        for g in range(P):  # equal share per GPU and layer
            add([(xv(j, i, g), 1.0) for i in range(E)], share, share)
        for i in range(E):  # one GPU per expert
            add([(xv(j, i, g), 1.0) for g in range(P)], 1, 1)
    for h, (j, i, p) in enumerate(hops):
        for g in range(P):
            add([(nx + h, 1.0), (xv(j, i, g), -1.0), (xv(j + 1, p, g), 1.0)], 0, np.inf)
            add([(nx + h, 1.0), (xv(j + 1, p, g), -1.0), (xv(j, i, g), 1.0)], 0, np.inf)
    res = milp(c, constraints=LinearConstraint(np.array(rows), lo, hi),
               integrality=np.ones(nv), bounds=Bounds(0, 1))
    if res.status != 0:
        raise RuntimeError(f"milp failed: {res.message}")
    x = np.round(res.x[:nx]).astype(np.int64).reshape(L, E, P)
    gpu_of = x.argmax(axis=2).astype(np.int32)
    return int(round(res.fun)), gpu_of


def greedy_order_makespan(D) -> int:
    """One list-schedule reading of the page's transmission-order steps (§Aurora 场景 1, the
    steps after 定理 4.2), for comparison with the bound only; the page does not fix these
    details, so other readings can end elsewhere. This reading: the bottleneck rank (largest
    send or receive volume) is scheduled first as a sender, even when its load is on the
    receive side (a rank that only receives then sends nothing and its own blocks are placed by
    the other senders like anyone else's); the other ranks follow by send volume, largest
    first; each rank sends its blocks one after another (largest first), each block whole (no
    pre-emption), starting at the earliest time at which both the rank and the block's
    receiver are free, so that no receiver is fed by two senders at once. Returns the time the
    last block ends, in rows (ties to the lower rank index)."""
    D = np.array(D, dtype=np.int64, copy=True)
    np.fill_diagonal(D, 0)
    W = D.shape[0]
    send, recv = D.sum(axis=1), D.sum(axis=0)
    load = np.maximum(send, recv)
    first = int(np.argmax(load))
    order = [first] + sorted((i for i in range(W) if i != first), key=lambda i: (-send[i], i))
    busy = [[] for _ in range(W)]   # per receiver: (start, end) intervals taken
    end_all = 0
    for i in order:
        t = 0
        for j in sorted((j for j in range(W) if D[i, j] > 0), key=lambda j: (-D[i, j], j)):
            n = int(D[i, j])
            start = t
            for a, b in sorted(busy[j]):   # first gap of length n at or after `start`
                if start + n <= a:
                    break
                start = max(start, b)
            busy[j].append((start, start + n))
            t = start + n
            end_all = max(end_all, t)
    return end_all
