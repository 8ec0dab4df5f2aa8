"""Brute-force restatement of the layer for tiny inputs, used to pin the oracle.

Independent of ``oracle/moe_oracle.c``: exact rational arithmetic for the fp32
fused multiply-add chain, a full sort for top-K, an O(N*K*E) recount for
positions, Python sets for deduplication and numpy float64 matmuls for the
expert FFN. Pure Python loops: tiny shapes only.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np


def _f32_bits(v: np.float32) -> int:
    return int(np.array(v, dtype=np.float32).view(np.uint32))


def round_to_f32(q: Fraction) -> float:
    """Round an exact rational to binary32, nearest with ties to even."""
    c0 = np.float32(float(q))
    cands = [np.nextafter(c0, np.float32(-np.inf)), c0, np.nextafter(c0, np.float32(np.inf))]
    best = None
    for c in cands:
        if not np.isfinite(c):
            continue
        dist = abs(Fraction(float(c)) - q)
        if (best is None or dist < best[0]
                or (dist == best[0] and (_f32_bits(c) & 1) == 0 and (_f32_bits(best[1]) & 1) == 1)):
            best = (dist, c)
    return float(best[1])


def fmaf_exact(a: float, b: float, c: float) -> float:
    return round_to_f32(Fraction(a) * Fraction(b) + Fraction(c))


def bf16_bits_to_float(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << 16).view(np.float32)


def logits(x_u16: np.ndarray, wr: np.ndarray, bias) -> np.ndarray:
    x = bf16_bits_to_float(x_u16)
    N, d = x.shape
    E = wr.shape[0]
    out = np.empty((N, E), np.float32)
    for t in range(N):
        for e in range(E):
            acc = 0.0
            for i in range(d):
                acc = fmaf_exact(float(x[t, i]), float(wr[e, i]), acc)
            if bias is not None:
                acc = round_to_f32(Fraction(acc) + Fraction(float(bias[e])))
            out[t, e] = acc
    return out


def topk(lg: np.ndarray, K: int):
    N, E = lg.shape
    idx = np.empty((N, K), np.int32)
    w = np.empty((N, K), np.float64)
    for t in range(N):
        order = sorted(range(E), key=lambda e: (-float(lg[t, e]), e))[:K]
        idx[t] = order
        ex = [math.exp(float(lg[t, e]) - float(lg[t, order[0]])) for e in order]
        s = math.fsum(ex)
        w[t] = [v / s for v in ex]
    return idx, w


def capacity(N: int, E: int, K: int, cf: float) -> int:
    if not cf > 0:
        return N * K
    return math.ceil(Fraction(cf) * N * K / E)


def dispatch(idx: np.ndarray, E: int, W: int, C: int, order: int = 0, reroute: bool = False,
             logits=None) -> dict:
    """order 0: priority by (token, slot); 1: by (slot, token). With ``reroute``, an
    overflowed assignment moves to the token's best remaining expert (by logit, then
    index) outside its top-K whose demand is below C, and queues behind that expert's
    first-pass assignments."""
    N, K = idx.shape
    flat = idx.reshape(-1)
    prio = (lambda a: a) if order == 0 else (lambda a: (a % K) * N + a // K)
    pos = [sum(1 for b in range(N * K) if flat[b] == flat[a] and prio(b) < prio(a))
           for a in range(N * K)]
    counts = [sum(1 for a in range(N * K) if flat[a] == e) for e in range(E)]
    expert_of = [int(flat[a]) if pos[a] < C else -1 for a in range(N * K)]
    if reroute:
        moved = {}
        for t in range(N):
            mine = {int(e) for e in idx[t]}
            cands = [e for e in sorted(range(E), key=lambda e: (-float(logits[t, e]), e))
                     if e not in mine and counts[e] < C]
            over = [t * K + k for k in range(K) if pos[t * K + k] >= C]
            for a, e in zip(over, cands):
                moved[a] = e
        for a, e in moved.items():
            p1 = counts[e] + sum(1 for b, e2 in moved.items() if e2 == e and prio(b) < prio(a))
            if p1 < C:
                expert_of[a] = e
                pos[a] = p1
    kept = [sum(1 for a in range(N * K) if expert_of[a] == e) for e in range(E)]
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + kept[e])
    row_of = [offsets[expert_of[a]] + pos[a] if expert_of[a] >= 0 else -1 for a in range(N * K)]
    e_per, n_per = E // W, N // W
    D = np.zeros((W, W), np.int64)
    keyed = []
    for a in range(N * K):
        if row_of[a] >= 0:
            t, e = a // K, expert_of[a]
            D[t // n_per, e // e_per] += 1
            keyed.append(((t // n_per, e // e_per, e, pos[a]), a))
    keyed.sort()
    packed_row_of = [-1] * (N * K)
    for p, (_, a) in enumerate(keyed):
        packed_row_of[a] = p
    dedup = 0
    for t in range(N):
        dests = {expert_of[t * K + k] // e_per for k in range(K) if expert_of[t * K + k] >= 0}
        dests.discard(t // n_per)
        dedup += len(dests)
    rerouted = sum(1 for a in range(N * K) if expert_of[a] >= 0 and expert_of[a] != flat[a])
    return dict(counts=np.array(counts), kept=np.array(kept), offsets=np.array(offsets),
                row_of=np.array(row_of), D=D, packed_row_of=np.array(packed_row_of), dedup=dedup,
                expert_of=np.array(expert_of), rerouted=rerouted)


def swiglu_rows(x_u16, w1_u16, w3_u16, w2_u16, row_token, row_expert):
    """Expert FFN through numpy float64 matmuls, one expert at a time."""
    x = bf16_bits_to_float(x_u16).astype(np.float64)
    w1 = bf16_bits_to_float(w1_u16).astype(np.float64)
    w3 = bf16_bits_to_float(w3_u16).astype(np.float64)
    w2 = bf16_bits_to_float(w2_u16).astype(np.float64)
    y = np.zeros((len(row_token), x.shape[1]))
    for e in sorted(set(int(v) for v in row_expert)):
        sel = np.nonzero(np.asarray(row_expert) == e)[0]
        X = x[np.asarray(row_token)[sel]]
        G = X @ w1[e].T
        U = X @ w3[e].T
        H = G / (1.0 + np.exp(-G)) * U
        y[sel] = H @ w2[e].T
    return y


def min_unit_slots(D) -> int:
    """Fewest unit time slots that carry the off-diagonal traffic of a small integer matrix D
    when, in one slot, every sender sends one row to at most one receiver and every receiver
    takes at most one row: breadth-first search over the remaining traffic."""
    D = np.array(D, dtype=np.int64)
    W = D.shape[0]
    np.fill_diagonal(D, 0)
    cells = [(i, j) for i in range(W) for j in range(W) if i != j]

    def matchings(rem):
        out = []

        def grow(k, used_r, used_c, chosen):
            if k == len(cells):
                if chosen:
                    out.append(tuple(chosen))
                return
            grow(k + 1, used_r, used_c, chosen)
            i, j = cells[k]
            if rem[i][j] > 0 and i not in used_r and j not in used_c:
                grow(k + 1, used_r | {i}, used_c | {j}, chosen + [(i, j)])

        grow(0, frozenset(), frozenset(), [])
        return out

    start = tuple(tuple(int(v) for v in r) for r in D)
    if not any(any(r) for r in start):
        return 0
    frontier, seen, depth = {start}, {start}, 0
    while frontier:
        depth += 1
        nxt = set()
        for s in frontier:
            for mt in matchings(s):
                rem = [list(r) for r in s]
                for i, j in mt:
                    rem[i][j] -= 1
                t = tuple(tuple(r) for r in rem)
                if not any(any(r) for r in t):
                    return depth
                if t not in seen:
                    seen.add(t)
                    nxt.add(t)
        frontier = nxt
    raise AssertionError("unreachable")


def balanced_placements(E: int, P: int):
    """Every assignment of E experts to P GPUs with E/P experts each."""
    share = E // P
    out = []

    def rec(e, load, cur):
        if e == E:
            out.append(tuple(cur))
            return
        for g in range(P):
            if load[g] < share:
                load[g] += 1
                cur.append(g)
                rec(e + 1, load, cur)
                cur.pop()
                load[g] -= 1

    rec(0, [0] * P, [])
    return out


def best_placement_cost(counts, P: int) -> int:
    """Exhaustive minimum over all balanced placements of every layer of the crossing hops."""
    import itertools
    counts = np.asarray(counts, dtype=np.int64)
    Lm1, E, _ = counts.shape
    opts = balanced_placements(E, P)
    best = None
    for combo in itertools.product(opts, repeat=Lm1 + 1):
        c = 0
        for j in range(Lm1):
            for i in range(E):
                for p in range(E):
                    if combo[j][i] != combo[j + 1][p]:
                        c += int(counts[j, i, p])
        best = c if best is None else min(best, c)
    return best
