"""Exchange planning on the host: the contention-free transmission order and the expert
placement of the C library against the oracle (CPU only; the functions need no GPU).

Pins of the oracle itself: the exchange bound against a breadth-first search for the fewest
unit slots (König's theorem says they agree), and the placement ILP against exhaustive search
over every balanced placement.
"""
from __future__ import annotations

import numpy as np
import pytest

import brute
from oracle import exchange_plan as xp

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


@pytest.fixture(scope="module")
def m():
    import combine_grouped_gemm_router_b200 as mod
    return mod


# ------------------------------------------------------------------ pins of the oracle

@pytest.mark.parametrize("seed", range(12))
def test_exchange_bound_is_the_fewest_unit_slots(seed):
    rng = np.random.default_rng(seed)
    W = 2 + seed % 2
    D = rng.integers(0, 3, (W, W))
    assert xp.exchange_bound(D) == brute.min_unit_slots(D)


def test_exchange_bound_hand_example():
    # off-diagonal row sums 2, 4, 8; column sums 5, 6, 3 -> the busiest rank sends 8 rows
    D = [[5, 2, 0], [1, 0, 3], [4, 4, 9]]
    assert xp.exchange_bound(D) == 8
    assert xp.exchange_bound([[7]]) == 0


@pytest.mark.parametrize("seed", range(6))
def test_placement_ilp_is_the_exhaustive_optimum(seed):
    rng = np.random.default_rng(100 + seed)
    L, E, P = [(2, 4, 2), (3, 4, 2), (2, 6, 3), (3, 6, 2), (2, 6, 2), (4, 4, 2)][seed]
    counts = rng.integers(0, 6, (L - 1, E, E))
    opt, g = xp.ilp_placement(counts, P)
    assert opt == brute.best_placement_cost(counts, P)
    assert xp.placement_cost(counts, g) == opt
    for layer in g:
        assert np.bincount(layer, minlength=P).tolist() == [E // P] * P


def test_placement_cost_hand_example():
    # two layers of 4 experts on 2 GPUs; expert 0 -> 2 (3 hops), 1 -> 3 (2 hops), 0 -> 0 (1 hop)
    counts = np.zeros((1, 4, 4), np.int64)
    counts[0, 0, 2], counts[0, 1, 3], counts[0, 0, 0] = 3, 2, 1
    contiguous = xp.contiguous_placement(2, 4, 2)        # {0,1} on GPU 0, {2,3} on GPU 1
    assert xp.placement_cost(counts, contiguous) == 5    # 0 -> 2 and 1 -> 3 cross
    swapped = np.array([[0, 0, 1, 1], [1, 1, 0, 0]])      # layer 1 mirrored
    assert xp.placement_cost(counts, swapped) == 1       # only 0 -> 0 crosses


# ------------------------------------------------------------------ the library

def check_schedule(D, dst, ln, span):
    D = np.asarray(D, dtype=np.int64)
    W = D.shape[0]
    assert dst.shape == (len(ln), W)
    assert (ln > 0).all()
    assert len(ln) <= 2 * W * W
    sent = np.zeros_like(D)
    for s in range(len(ln)):
        d = dst[s]
        busy = d[d >= 0]
        assert len(set(busy.tolist())) == len(busy), "a receiver fed by two senders"
        assert all(d[i] != i for i in range(W))
        assert ((d >= -1) & (d < W)).all()
        for i in range(W):
            if d[i] >= 0:
                sent[i, d[i]] += ln[s]
        if s > 0:
            assert (dst[s] != dst[s - 1]).any(), "equal neighbouring phases are merged"
    off = D.copy()
    np.fill_diagonal(off, 0)
    assert (sent == off).all()
    assert int(ln.sum()) == span


SCHEDULE_CASES = [
    ("one_rank", lambda r: np.array([[9]])),
    ("zeros", lambda r: np.zeros((8, 8), np.int64)),
    ("diagonal_only", lambda r: np.diag(r.integers(1, 50, 8))),
    ("uniform_8", lambda r: r.integers(0, 1000, (8, 8))),
    ("skewed_8", lambda r: (r.integers(0, 100, (8, 8)) * (np.arange(8) + 1) ** 2)),
    ("one_hot_receiver", lambda r: np.outer(r.integers(1, 9, 8), np.eye(8)[3]).astype(np.int64)),
    ("sparse_16", lambda r: r.integers(0, 50, (16, 16)) * (r.random((16, 16)) < 0.2)),
    ("dense_64", lambda r: r.integers(0, 10000, (64, 64))),
    ("two_ranks", lambda r: np.array([[3, 11], [4, 0]])),
]


@pytest.mark.parametrize("name,make", SCHEDULE_CASES, ids=[c[0] for c in SCHEDULE_CASES])
def test_exchange_schedule_reaches_the_bound(m, name, make):
    D = make(np.random.default_rng(7))
    dst, ln, span = m.moe_exchange_schedule(D)
    assert span == xp.exchange_bound(D)
    check_schedule(D, dst, ln, span)


def test_exchange_schedule_phases_are_few(m):
    """Phases chosen by their shortest transfer (largest first) stay few: on dense matrices a
    small multiple of W, far below the 2*W*W that any decomposition stays under."""
    rng = np.random.default_rng(1)
    for W in (8, 16, 64):
        D = rng.integers(0, 1000, (W, W))
        _, ln, _ = m.moe_exchange_schedule(D)
        assert len(ln) <= 5 * W, (W, len(ln))


def test_exchange_schedule_on_dispatch_traffic(m):
    """The traffic matrix of a real routing (oracle positions of a skewed top-8 routing)."""
    import oracle
    rng = np.random.default_rng(3)
    N, E, K, W = 512, 32, 4, 8
    logits = rng.standard_normal((N, E)) - 0.8 * np.log1p(np.arange(E))
    idx = np.argsort(-logits, axis=1, kind="stable")[:, :K].astype(np.int32)
    for C in (N * K, 40):
        D = oracle.positions(idx, E, W, C)["D"].reshape(W, W)
        dst, ln, span = m.moe_exchange_schedule(D)
        assert span == xp.exchange_bound(D)
        check_schedule(D, dst, ln, span)


def test_exchange_schedule_errors(m):
    D = np.random.default_rng(0).integers(1, 9, (8, 8))
    with pytest.raises(m.MoeError):
        m.moe_exchange_schedule(D, max_phases=1)     # the order needs more phases
    bad = D.copy()
    bad[1, 2] = -1
    with pytest.raises(m.MoeError):
        m.moe_exchange_schedule(bad)
    with pytest.raises(m.MoeError):
        m.moe_exchange_schedule(np.zeros((65, 65), np.int64))


@pytest.mark.parametrize("seed", range(8))
def test_placement_valid_and_costed(m, seed):
    rng = np.random.default_rng(200 + seed)
    L, E, P = [(2, 8, 2), (3, 8, 4), (4, 16, 4), (2, 64, 8), (4, 64, 8), (3, 32, 8),
               (2, 8, 8), (3, 12, 3)][seed]
    counts = rng.integers(0, 20, (L - 1, E, E))
    g, cost, base = m.moe_place_experts(counts, L, E, P, starts=4)
    for layer in g:
        assert np.bincount(layer, minlength=P).tolist() == [E // P] * P
    assert cost == xp.placement_cost(counts, g)
    assert base == xp.placement_cost(counts, xp.contiguous_placement(L, E, P))
    assert cost <= base


@pytest.mark.parametrize("seed", range(10))
def test_placement_matches_the_ilp_on_small_layers(m, seed):
    """The local search never beats the ILP's optimum (a check of both), and with 8 starts it
    reaches that optimum on each of these seeded random stacks. That is a property of these
    instances, not a guarantee of the method (one start can stop well above it)."""
    rng = np.random.default_rng(300 + seed)
    L, E, P = [(2, 4, 2), (3, 4, 2), (2, 6, 2), (3, 6, 3), (2, 8, 2), (3, 8, 2), (2, 8, 4),
               (4, 6, 2), (3, 8, 4), (2, 9, 3)][seed]
    counts = rng.integers(0, 10, (L - 1, E, E))
    opt, _ = xp.ilp_placement(counts, P)
    _, one, _ = m.moe_place_experts(counts, L, E, P, starts=1)
    assert opt <= one
    _, cost, _ = m.moe_place_experts(counts, L, E, P, starts=8)
    assert cost == opt


def test_placement_recovers_planted_affinity(m):
    """Layers whose experts hand tokens on to one partner expert each (a permutation per layer
    pair, with a little noise): the best placement keeps every partner pair on one GPU."""
    rng = np.random.default_rng(11)
    L, E, P = 4, 64, 8
    counts = rng.integers(0, 2, (L - 1, E, E))
    planted = 0
    for j in range(L - 1):
        perm = rng.permutation(E)
        counts[j, np.arange(E), perm] += 500
        planted += 500 * E
    g, cost, base = m.moe_place_experts(counts, L, E, P, starts=4)
    noise = int(counts.sum()) - planted
    assert cost <= noise                    # no planted hop crosses GPUs
    assert base > 0.8 * planted * (1 - 1 / P)


def test_placement_degenerate_shapes(m):
    g, cost, base = m.moe_place_experts(np.zeros(0, np.int64), 1, 8, 2)
    assert g.tolist() == [[0, 0, 0, 0, 1, 1, 1, 1]] and cost == 0 and base == 0
    g, cost, base = m.moe_place_experts(np.ones((1, 4, 4), np.int64), 2, 4, 1)
    assert (g == 0).all() and cost == 0 and base == 0
    g, cost, base = m.moe_place_experts(np.ones((1, 4, 4), np.int64), 2, 4, 4)
    assert cost == base == 12          # one expert per GPU: 4 of the 16 hops stay


def test_placement_errors(m):
    c = np.ones((1, 8, 8), np.int64)
    for args in [(c, 2, 8, 3), (c, 2, 8, 0), (-c, 2, 8, 2)]:
        with pytest.raises(m.MoeError):
            m.moe_place_experts(*args)
    with pytest.raises(m.MoeError):
        m.moe_place_experts(c, 2, 8, 2, starts=0)
    with pytest.raises(m.MoeError):
        m.moe_place_experts(np.ones((1, 300, 300), np.int64), 2, 300, 2)


def test_placement_deployed_by_relabelling_experts(m):
    """Deploying a placement = storing each layer's experts GPU by GPU (router rows permuted
    with them). The routing is the same up to the relabelling, and the relabelled stack's
    affinity counts under the contiguous placement cost exactly what moe_place_experts
    reported: the placement's cost is the crossing count the deployed layers will show."""
    import torch

    import oracle
    from moe_workloads import WORKLOADS, affine_router
    w = WORKLOADS["stack4_affinity"].with_(N=256, d=64, f=128, E=16, K=2, W=4, layers=3)
    L, E, K, P = w.layers, w.E, w.K, w.W
    g = torch.Generator().manual_seed(4)
    x0 = torch.randn(w.N, w.d, generator=g)
    xs = [(x0 + 0.3 * torch.randn(w.N, w.d, generator=g)).to(torch.bfloat16) for _ in range(L)]
    routers = [affine_router(w, 0, l) for l in range(L)]
    topk = [oracle.topk(oracle.router_logits(xs[l], routers[l]), K)[0] for l in range(L)]
    counts = np.stack([oracle.affinity(topk[j], topk[j + 1], E) for j in range(L - 1)])
    gpu_of, cost, base = m.moe_place_experts(counts, L, E, P)
    assert cost < base
    topk2, new_ids = [], []
    orders = m.placement_order(gpu_of, P)
    for l in range(L):
        order = orders[l]                                   # GPU by GPU, experts ascending
        assert (gpu_of[l][order] == np.arange(E) // (E // P)).all()
        new_id = np.empty(E, np.int64)
        new_id[order] = np.arange(E)
        new_ids.append(new_id)
        t2 = oracle.topk(oracle.router_logits(xs[l], routers[l][torch.from_numpy(order)]), K)[0]
        np.testing.assert_array_equal(t2, new_id[topk[l]])  # same choices, new names
        topk2.append(t2)
    counts2 = np.stack([oracle.affinity(topk2[j], topk2[j + 1], E) for j in range(L - 1)])
    for j in range(L - 1):
        np.testing.assert_array_equal(counts2[j][np.ix_(new_ids[j], new_ids[j + 1])], counts[j])
    assert xp.placement_cost(counts2, xp.contiguous_placement(L, E, P)) == cost


@pytest.mark.parametrize("seed", range(4))
def test_staged_placement_costs_and_shape(m, seed):
    """Nodes first, then GPUs inside each node: every GPU holds E / (nodes * gpus) experts of
    every layer; the reported node and GPU hop counts are the oracle's costs of the placement
    seen at node and at GPU granularity; stage 1 is moe_place_experts on the nodes."""
    rng = np.random.default_rng(400 + seed)
    L, E, nodes, gpn = [(3, 16, 2, 4), (4, 32, 4, 2), (2, 64, 2, 4), (3, 24, 3, 2)][seed]
    counts = rng.integers(0, 12, (L - 1, E, E))
    g, hops = m.moe_place_experts_staged(counts, L, E, nodes, gpn, starts=4)
    P = nodes * gpn
    for layer in g:
        assert np.bincount(layer, minlength=P).tolist() == [E // P] * P
    assert hops["gpu_hops"] == xp.placement_cost(counts, g)
    assert hops["node_hops"] == xp.placement_cost(counts, g // gpn)
    contiguous = xp.contiguous_placement(L, E, P)
    assert hops["contiguous_gpu_hops"] == xp.placement_cost(counts, contiguous)
    assert hops["contiguous_node_hops"] == xp.placement_cost(counts, contiguous // gpn)
    _, node_cost, _ = m.moe_place_experts(counts, L, E, nodes, starts=4)
    assert hops["node_hops"] == node_cost
    assert hops["node_hops"] <= hops["contiguous_node_hops"]


def test_staged_placement_keeps_planted_groups_on_nodes(m):
    """Tokens that stay inside groups of 8 experts across layers (a permutation of the groups
    per layer, plus noise): the staged placement keeps every group on one node, so the only
    node crossings are the noise; inside the node the hops between the group's experts also
    follow a partner permutation, which stage 2 keeps on one GPU."""
    rng = np.random.default_rng(12)
    L, E, nodes, gpn = 3, 32, 4, 2
    counts = rng.integers(0, 2, (L - 1, E, E))
    planted = 0
    groups = rng.permutation(E).reshape(nodes, E // nodes)   # layer 0's groups
    for j in range(L - 1):
        perm = rng.permutation(E)        # expert i hands on to perm[i] ...
        for grp in groups:               # ... and to the rest of its group's image, less so
            nxt = perm[grp]
            for a in grp:
                counts[j, a, nxt] += 20
                planted += 20 * len(nxt)
            counts[j, grp, nxt] += 200
            planted += 200 * len(grp)
        groups = perm[groups]            # the groups of layer j + 1
    g, hops = m.moe_place_experts_staged(counts, L, E, nodes, gpn, starts=8)
    noise = int(counts.sum()) - planted
    assert hops["node_hops"] <= noise
    assert hops["gpu_hops"] < 0.5 * hops["contiguous_gpu_hops"]


def test_staged_placement_errors(m):
    c = np.ones((1, 12, 12), np.int64)
    with pytest.raises(m.MoeError):
        m.moe_place_experts_staged(c, 2, 12, 5, 2)    # 12 experts do not split over 10 GPUs
    with pytest.raises(m.MoeError):
        m.moe_place_experts_staged(-c, 2, 12, 2, 3)


def test_placement_order_errors(m):
    with pytest.raises(m.MoeError):
        m.placement_order(np.array([[0, 0, 0, 1]]), 2)   # GPU 0 holds 3 of 4 experts
    with pytest.raises(m.MoeError):
        m.placement_order(np.array([[0, 2, 1, 1]]), 2)   # no GPU 2
    assert m.placement_order(np.array([[1, 0, 0, 1]]), 2).tolist() == [[1, 2, 0, 3]]


def test_schedule_on_random_and_degenerate_matrices(m):
    """Seeded sweep: tiny entries (many ties), huge sparse entries (2^40), one non-zero block,
    rank-one traffic, dense traffic, 1 to 19 ranks; every order a valid contention-free
    delivery of D of length tau_min."""
    rng = np.random.default_rng(123)
    for it in range(120):
        W = int(rng.integers(1, 20))
        kind = it % 5
        if kind == 0:
            D = rng.integers(0, 3, (W, W))
        elif kind == 1:
            D = (rng.integers(0, 2 ** 40, (W, W)) * (rng.random((W, W)) < 0.3)).astype(np.int64)
        elif kind == 2:
            D = np.zeros((W, W), np.int64)
            D[rng.integers(0, W), rng.integers(0, W)] = int(rng.integers(1, 100))
        elif kind == 3:
            D = np.outer(rng.integers(0, 5, W), rng.integers(0, 5, W)).astype(np.int64)
        else:
            D = rng.integers(0, 1000, (W, W))
        dst, ln, span = m.moe_exchange_schedule(D)
        assert span == xp.exchange_bound(D)
        if len(ln):
            check_schedule(D, dst, ln, span)


def test_placements_on_random_and_degenerate_counts(m):
    """Seeded sweep of one-level and staged placements: no hops at all, 0/1 counts, counts up
    to 1e9; shapes, costs (oracle), never worse than contiguous, and the storage order."""
    rng = np.random.default_rng(7)
    for it in range(60):
        P, share, L = int(rng.integers(1, 6)), int(rng.integers(1, 5)), int(rng.integers(1, 5))
        E = P * share
        hi = (1, 2, 10 ** 9)[it % 3]
        c = rng.integers(0, hi, (L - 1, E, E)) if L > 1 else np.zeros(0, np.int64)
        g, cost, base = m.moe_place_experts(c, L, E, P, starts=3)
        for row in g:
            assert np.bincount(row, minlength=P).tolist() == [share] * P
        if L > 1:
            assert cost == xp.placement_cost(c, g) <= base
            assert base == xp.placement_cost(c, xp.contiguous_placement(L, E, P))
        order = m.placement_order(g, P)
        assert all((g[l][order[l]] == np.arange(E) // share).all() for l in range(L))
        if P > 1 and P % 2 == 0:
            gs, hops = m.moe_place_experts_staged(c, L, E, 2, P // 2, starts=2)
            if L > 1:
                assert hops["gpu_hops"] == xp.placement_cost(c, gs)
                assert hops["node_hops"] == xp.placement_cost(c, gs // (P // 2))


def test_literal_greedy_reading_misses_the_bound():
    """One list-schedule reading of the page's steps (whole blocks, bottleneck rank first as a
    sender, the rest by volume, each block at the earliest time its receiver is free) never
    beats tau_min (no order can) and, in this reading, on random 8-rank traffic ends well above
    it (the 0.2 mean-gap threshold belongs to this reading only); the library builds its order
    by a matching decomposition that meets the bound exactly."""
    rng = np.random.default_rng(0)
    gaps = []
    for _ in range(100):
        D = rng.integers(0, 1000, (8, 8)) * (rng.random((8, 8)) < 0.8)
        bound = xp.exchange_bound(D)
        g = xp.greedy_order_makespan(D)
        assert g >= bound
        gaps.append(g / bound - 1)
    assert np.mean(gaps) > 0.2
    # a hand-checked case: 0 -> 1 (2 rows), 0 -> 2 (1), 1 -> 2 (2), 2 -> 0 (1). tau_min = 3
    # (rank 0 sends 3, rank 2 receives 3); whole blocks, largest first: 0 sends to 1 over [0, 2)
    # then to 2 over [2, 3); rank 1 (next by volume) sends to 2 over [0, 2); rank 2 to 0 over
    # [0, 1): makespan 3, the bound.
    D = np.array([[0, 2, 1], [0, 0, 2], [1, 0, 0]])
    assert xp.exchange_bound(D) == 3 and xp.greedy_order_makespan(D) == 3
