"""Pins of the CPU oracle against things other than itself: hand-worked
fixtures, brute force on tiny inputs, closed forms, library routines and
invariants. CPU only."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import brute
from moe_workloads import Workload, WORKLOADS, make_layer_inputs, random_small_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


# --------------------------------------------------------------------------- hand-worked

def test_hand_routing_fixture(orc):
    g = _load("hand_routing.json")
    lg = np.array(g["logits"], np.float32)
    idx, w, bad = orc.topk(lg, g["K"])
    assert bad == 0
    np.testing.assert_array_equal(idx, g["topk_idx"])
    np.testing.assert_allclose(w, g["topk_w"], rtol=1e-6, atol=0)
    C = orc.capacity(g["N"], g["E"], g["K"], g["cf"])
    assert C == g["C"]
    p = orc.positions(idx, g["E"], g["W"], C)
    for key in ("counts", "kept", "offsets", "row_of", "assign_of_row", "pk_off", "packed_row_of"):
        np.testing.assert_array_equal(p[key], g[key], err_msg=key)
    np.testing.assert_array_equal(p["D"], g["D"])
    assert {k: p["stats"][k] for k in g["stats"]} == g["stats"]
    assert p["stats"]["rerouted"] == 0  # no re-routing unless asked
    rep = orc.derive_report(g["N"], g["E"], g["K"], g["W"], p["kept"], p["D"], p["stats"], d=1)
    for key, v in g["report"].items():
        assert rep[key] == pytest.approx(v, rel=1e-12), key


def test_dispatch_volume_worked_example(orc):
    g = _load("dispatch_volume.json")
    for c in g["cases"]:
        b = orc.dispatch_bytes(c["rows"], g["d"], g["elem_bytes"])
        assert b == c["bytes"], c["name"]
        assert abs(b - c["printed_value"]) <= c["rel_round"] * c["printed_value"], c["name"]


def test_dispatch_volume_through_routing(orc):
    # K=1 dropless routing of 2048 tokens at d=2048 carries the prefill figure
    rng = np.random.default_rng(0)
    lg = rng.standard_normal((2048, 16)).astype(np.float32)
    idx, _, _ = orc.topk(lg, 1)
    p = orc.positions(idx, 16, 4, orc.capacity(2048, 16, 1, 0.0))
    rep = orc.derive_report(2048, 16, 1, 4, p["kept"], p["D"], p["stats"], d=2048, elem_bytes=2)
    assert rep["dispatch_bytes"] == 8388608


# --------------------------------------------------------------------------- brute force

def _tiny_inputs(w: Workload, seed: int):
    inp = make_layer_inputs(w, seed=seed)
    return inp


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_tiny(orc, seed):
    rng = torch.Generator().manual_seed(100 + seed)
    w = random_small_workload(rng, max_n=16, max_e=8)
    inp = _tiny_inputs(w, seed)
    xu = orc.as_u16(inp["x"])
    wr = inp["w_router"].numpy()
    bias = None if inp["bias"] is None else inp["bias"].numpy()

    # logits: exact rational fmaf chain vs the oracle, bit for bit
    lg_b = brute.logits(xu, wr, bias)
    lg_o = orc.router_logits(inp["x"], inp["w_router"], inp["bias"])
    np.testing.assert_array_equal(lg_o.view(np.uint32), lg_b.view(np.uint32))

    # top-K by a full sort; weights by fp64 softmax
    idx_b, w_b = brute.topk(lg_b, w.K)
    idx_o, w_o, bad = orc.topk(lg_o, w.K)
    assert bad == 0
    np.testing.assert_array_equal(idx_o, idx_b)
    np.testing.assert_allclose(w_o, w_b, rtol=2e-7, atol=0)

    C = orc.capacity(w.N, w.E, w.K, w.cf)
    assert C == brute.capacity(w.N, w.E, w.K, w.cf)
    p = orc.positions(idx_o, w.E, w.W, C)
    b = brute.dispatch(idx_b, w.E, w.W, C)
    for key in ("counts", "kept", "offsets", "row_of", "packed_row_of"):
        np.testing.assert_array_equal(p[key], b[key], err_msg=key)
    np.testing.assert_array_equal(p["D"], b["D"])
    assert p["stats"]["dedup_pairs"] == b["dedup"]

    # whole layer output vs numpy float64 matmul experts + a Python combine
    r = orc.layer(inp, w.K, w.W, w.cf)
    aor = r["assign_of_row"]
    y_b = brute.swiglu_rows(xu, orc.as_u16(inp["w1"]), orc.as_u16(inp["w3"]), orc.as_u16(inp["w2"]),
                            aor // w.K, idx_b.reshape(-1)[aor])
    np.testing.assert_allclose(r["y_rows"], y_b, rtol=1e-10, atol=1e-13)
    out_b = np.zeros((w.N, w.d))
    for t in range(w.N):
        for k in range(w.K):
            row = b["row_of"][t * w.K + k]
            if row >= 0:
                out_b[t] += float(w_o[t, k]) * y_b[row]
    np.testing.assert_allclose(r["out"], out_b, rtol=1e-10, atol=1e-13)


def test_brute_force_tiny_workload(orc):
    """The 'tiny' workload, logits and routing checked by brute force."""
    w = WORKLOADS["tiny"]
    inp = make_layer_inputs(w, seed=0)
    xu = orc.as_u16(inp["x"])
    # brute-force logits on a token subset (exact rational arithmetic is slow)
    sub = slice(0, 6)
    lg_b = brute.logits(xu[sub], inp["w_router"].numpy(), None)
    lg_o = orc.router_logits(inp["x"], inp["w_router"], None)
    np.testing.assert_array_equal(lg_o[sub].view(np.uint32), lg_b.view(np.uint32))
    idx_o, _, _ = orc.topk(lg_o, w.K)
    idx_b, _ = brute.topk(lg_o, w.K)
    np.testing.assert_array_equal(idx_o, idx_b)
    p = orc.positions(idx_o, w.E, w.W, orc.capacity(w.N, w.E, w.K, w.cf))
    b = brute.dispatch(idx_b, w.E, w.W, orc.capacity(w.N, w.E, w.K, w.cf))
    np.testing.assert_array_equal(p["row_of"], b["row_of"])
    np.testing.assert_array_equal(p["packed_row_of"], b["packed_row_of"])


# --------------------------------------------------------------------------- special cases

def test_single_expert_is_dense_swiglu(orc):
    """E = 1, K = 1: the layer is the dense SwiGLU FFN, gate weight exactly 1."""
    w = Workload("dense", N=24, d=64, f=96, E=1, K=1, W=1)
    inp = make_layer_inputs(w, seed=3)
    r = orc.layer(inp, 1, 1, 0.0)
    assert np.all(r["topk_w"] == 1.0)
    x = brute.bf16_bits_to_float(orc.as_u16(inp["x"])).astype(np.float64)
    w1 = brute.bf16_bits_to_float(orc.as_u16(inp["w1"]))[0].astype(np.float64)
    w3 = brute.bf16_bits_to_float(orc.as_u16(inp["w3"]))[0].astype(np.float64)
    w2 = brute.bf16_bits_to_float(orc.as_u16(inp["w2"]))[0].astype(np.float64)
    g = x @ w1.T
    u = x @ w3.T
    dense = (g * (1.0 / (1.0 + np.exp(-g))) * u) @ w2.T
    np.testing.assert_allclose(r["out"], dense, rtol=1e-10, atol=1e-14)


def test_swiglu_closed_form(orc):
    """One-hot input: g_j = W1[j][0], u_j = W3[j][0] exactly, so
    h_j = g_j * sigmoid(g_j) * u_j and y_i = sum_j h_j W2[i][j] in closed form."""
    d, f = 8, 4
    x = torch.zeros(1, d, dtype=torch.bfloat16)
    x[0, 0] = 1.0
    gvals = [-2.0, -0.5, 0.0, 3.0]
    uvals = [1.5, -1.0, 2.0, 0.25]
    w1 = torch.zeros(1, f, d, dtype=torch.bfloat16)
    w3 = torch.zeros(1, f, d, dtype=torch.bfloat16)
    w2 = torch.zeros(1, d, f, dtype=torch.bfloat16)
    for j in range(f):
        w1[0, j, 0] = gvals[j]
        w3[0, j, 0] = uvals[j]
    w2[0, 1, :] = torch.tensor([1.0, 2.0, -1.0, 0.5], dtype=torch.bfloat16)
    h, y = orc.expert_rows(np.array([0]), np.array([0]), x, w1, w3, w2, want_h=True)
    h_ref = [g / (1.0 + math.exp(-g)) * u for g, u in zip(gvals, uvals)]
    np.testing.assert_allclose(h[0], h_ref, rtol=1e-15)
    y_ref = np.zeros(d)
    y_ref[1] = h_ref[0] * 1.0 + h_ref[1] * 2.0 - h_ref[2] + h_ref[3] * 0.5
    np.testing.assert_allclose(y[0], y_ref, rtol=1e-15, atol=1e-300)


def test_identity_experts_round_trip(orc):
    """Identity experts (y row = the dispatched x row): combine(dispatch(x))
    returns x * sum of kept weights; dropless, that sum is 1 up to fp32 weight
    rounding."""
    for cf in (0.0, 0.75):
        w = Workload("id", N=64, d=32, f=8, E=8, K=3, W=4, cf=cf, s=1.1)
        inp = make_layer_inputs(w, seed=7)
        r = orc.route_and_dispatch(inp["x"], inp["w_router"], inp["bias"], w.K, w.W, w.cf)
        x = brute.bf16_bits_to_float(orc.as_u16(inp["x"])).astype(np.float64)
        y_rows = x[r["assign_of_row"] // w.K]
        y_of_slot = np.zeros((w.N * w.K, w.d))
        kept = r["row_of"] >= 0
        y_of_slot[kept] = y_rows[r["row_of"][kept]]
        out = orc.combine(r["row_of"], r["topk_w"], y_of_slot)
        wsum = np.where(r["row_of"].reshape(w.N, w.K) >= 0, r["topk_w"].astype(np.float64), 0).sum(1)
        np.testing.assert_allclose(out, x * wsum[:, None], rtol=1e-12, atol=1e-15)
        if cf == 0.0:
            np.testing.assert_allclose(wsum, 1.0, rtol=0, atol=4e-7)
        else:
            assert r["stats"]["dropped"] > 0


def test_fully_dropped_token_outputs_zero(orc):
    lg = np.array([[1.0, 0.0], [1.0, 0.0], [1.0, 0.0]], np.float32)  # all pick expert 0
    idx, wts, _ = orc.topk(lg, 1)
    p = orc.positions(idx, 2, 1, 2)
    assert list(p["row_of"]) == [0, 1, -1]
    out = orc.combine(p["row_of"], wts, np.ones((3, 4)))
    np.testing.assert_array_equal(out[2], 0.0)
    np.testing.assert_array_equal(out[:2], 1.0)


def test_ties_and_signed_zero(orc):
    lg = np.array([[0.0, -0.0, 0.0, -1.0], [2.0, 2.0, 2.0, 2.0]], np.float32)
    idx, w, _ = orc.topk(lg, 3)
    assert idx.tolist() == [[0, 1, 2], [0, 1, 2]]
    np.testing.assert_allclose(w[1], [1 / 3] * 3, rtol=1e-7)


def test_nonfinite_logit_counted(orc):
    lg = np.array([[0.0, np.nan], [1.0, 2.0], [np.inf, 0.0]], np.float32)
    _, _, bad = orc.topk(lg, 1)
    assert bad == 2


def test_capacity_exact():
    import oracle
    cases = [(8192, 128, 8, 1.25, 640), (32768, 64, 6, 1.0, 3072), (32768, 64, 6, 1.25, 3840),
             (32768, 64, 6, 2.0, 6144), (4, 4, 2, 1.0, 2), (10, 3, 2, 1.0, 7), (7, 5, 3, 0.3, 2)]
    for N, E, K, cf, want in cases:
        assert oracle.capacity(N, E, K, cf) == want == math.ceil(Fraction(cf) * N * K / E)
    assert oracle.capacity(16, 256, 8, 0.0) == 16 * 8


# --------------------------------------------------------------------------- invariants

@pytest.mark.parametrize("name,cf,s", [("e128_skew", 1.25, 1.1), ("stack4", 1.0, 1.2),
                                        ("stack4", 2.0, 0.0)])
def test_routing_invariants_at_scale(orc, name, cf, s):
    """Integer invariants on full-size routing (logits drawn directly; the
    invariants do not depend on how the logits arose)."""
    w = WORKLOADS[name].with_(cf=cf, s=s)
    rng = np.random.default_rng(11)
    lg = rng.standard_normal((w.N, w.E)).astype(np.float32)
    if s:
        lg = lg + np.array([-s * math.log(e + 1) for e in range(w.E)], np.float32)
    idx, wts, _ = orc.topk(lg, w.K)
    C = orc.capacity(w.N, w.E, w.K, w.cf)
    p = orc.positions(idx, w.E, w.W, C)
    NK = w.N * w.K
    assert p["counts"].sum() == NK
    assert p["kept"].sum() == NK - p["stats"]["dropped"] == p["R"]
    assert p["kept"].max() <= C
    np.testing.assert_array_equal(p["counts"], np.bincount(idx.reshape(-1), minlength=w.E))
    # every kept (t, k) exactly once among the rows; each token K - drops times
    aor = p["assign_of_row"]
    assert len(np.unique(aor)) == p["R"]
    np.testing.assert_array_equal(p["row_of"][aor], np.arange(p["R"]))
    drops = (p["row_of"].reshape(w.N, w.K) < 0).sum(1)
    np.testing.assert_array_equal(np.bincount(aor // w.K, minlength=w.N), w.K - drops)
    # rows inside each expert come in increasing token order
    rows_e = idx.reshape(-1)[aor]
    assert np.all(np.diff(rows_e) >= 0)
    same = rows_e[1:] == rows_e[:-1]
    assert np.all(np.diff(aor)[same] > 0)
    # traffic matrix and packing
    assert p["D"].sum() == p["R"]
    assert p["pk_off"][-1] == p["R"]
    pk = p["packed_row_of"][p["row_of"] >= 0]
    assert sorted(pk.tolist()) == list(range(p["R"]))
    # per-home-rank rows = row sums of D
    home = (aor // w.K) // (w.N // w.W)
    np.testing.assert_array_equal(np.bincount(home, minlength=w.W), p["D"].sum(1))


def test_mean_send_volume_closed_form(orc):
    """Dropless, the mean per-rank send equals N*K*d*b/W
    [MoE 专家并行的 All-to-All 通信瓶颈, §专家越多，通信为什么越重]."""
    N, E, K, W, d = 4096, 64, 6, 8, 4096
    rng = np.random.default_rng(5)
    idx, _, _ = orc.topk(rng.standard_normal((N, E)).astype(np.float32), K)
    p = orc.positions(idx, E, W, orc.capacity(N, E, K, 0.0))
    send_bytes = p["D"].sum(1) * d * 2
    assert send_bytes.mean() == N * K * d * 2 / W


def test_local_fraction_is_one_over_w(orc):
    """Unbiased routing with experts spread evenly: a routed row stays on its
    home rank with probability (E/W)/E = 1/W
    [MoE 专家并行的 All-to-All 通信瓶颈, §专家越多，通信为什么越重]."""
    N, E, K, W = 8192, 64, 6, 8
    rng = np.random.default_rng(9)
    idx, _, _ = orc.topk(rng.standard_normal((N, E)).astype(np.float32), K)
    p = orc.positions(idx, E, W, orc.capacity(N, E, K, 0.0))
    local = np.trace(p["D"]) / p["R"]
    n = p["R"]
    sigma = math.sqrt((1 / W) * (1 - 1 / W) / n) * math.sqrt(K)  # slots of a token correlate
    assert abs(local - 1 / W) < 4 * sigma
    rep = orc.derive_report(N, E, K, W, p["kept"], p["D"], p["stats"], d=1)
    assert rep["cross_rank_fraction"] == pytest.approx(1 - local)


def test_tau_min_identity(orc):
    """Aurora's bound on a hand traffic matrix: the busiest sender or receiver
    [MoE Inference Communication, §Aurora 定理 4.2]."""
    D = np.array([[5, 2, 0], [1, 7, 4], [3, 0, 2]])
    rep = orc.derive_report(3, 3, 1, 3, np.array([1, 1, 1]), D,
                            dict(R=int(D.sum()), dropped=0, cross_rows=10, dedup_pairs=0,
                                 active_experts=3), d=1)
    # off-diagonal row sums 2, 5, 3; column sums 4, 2, 4
    assert rep["tau_min_tokens"] == 5
    assert rep["send_max"] == 12 and rep["recv_min"] == 6


def test_affinity_invariants(orc):
    """Affinity counts [MoE Inference Communication, §ExFlow 跨层专家亲和性]:
    brute-force recount, row sums K * n_j(i), total K^2 N."""
    N, E, K = 300, 16, 3
    rng = np.random.default_rng(4)
    a, _, _ = orc.topk(rng.standard_normal((N, E)).astype(np.float32), K)
    b, _, _ = orc.topk(rng.standard_normal((N, E)).astype(np.float32), K)
    cnt = orc.affinity(a, b, E)
    ref = np.zeros((E, E), np.int64)
    for t in range(N):
        for i in a[t]:
            for p_ in b[t]:
                ref[i, p_] += 1
    np.testing.assert_array_equal(cnt, ref)
    n_i = np.bincount(a.reshape(-1), minlength=E)
    np.testing.assert_array_equal(cnt.sum(1), K * n_i)
    assert cnt.sum() == K * K * N
    # identical consecutive routing: mass on the K x K blocks of each token
    same = orc.affinity(a, a, E)
    assert np.trace(same) == N * K


def test_sampled_layer_matches_full(orc):
    w = Workload("s", N=48, d=64, f=64, E=8, K=2, W=4, cf=1.0, s=1.1)
    inp = make_layer_inputs(w, seed=2)
    full = orc.layer(inp, w.K, w.W, w.cf)
    toks = [0, 5, 17, 47]
    smp = orc.layer_sampled(inp, w.K, w.W, w.cf, toks)
    np.testing.assert_allclose(smp["out_tokens"], full["out"][toks], rtol=1e-13, atol=1e-15)


def test_residual_moe_oracle(orc):
    """Residual-MoE [MoE Inference Communication, §PR-MoE]: the shared dense MLP equals a numpy
    float64 SwiGLU on every token, and the layer output is the routed output plus it: with the
    routed experts' down projections zeroed the layer is exactly the dense MLP."""
    from moe_workloads import make_shared_inputs
    w = Workload("res", N=40, d=64, f=64, E=4, K=1, W=2, shared_f=96)
    inp = make_layer_inputs(w, seed=4)
    sh = make_shared_inputs(w, seed=4)
    r = orc.layer_shared(inp, sh, w.K, w.W, w.cf)
    x = brute.bf16_bits_to_float(orc.as_u16(inp["x"])).astype(np.float64)
    a = brute.bf16_bits_to_float(orc.as_u16(sh["ws1"])).astype(np.float64)
    b = brute.bf16_bits_to_float(orc.as_u16(sh["ws3"])).astype(np.float64)
    c = brute.bf16_bits_to_float(orc.as_u16(sh["ws2"])).astype(np.float64)
    g, u = x @ a.T, x @ b.T
    dense = (g / (1.0 + np.exp(-g)) * u) @ c.T
    np.testing.assert_allclose(r["shared_y"], dense, rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(r["out"], r["out_routed"] + dense, rtol=1e-12, atol=1e-15)
    assert np.all(r["topk_w"] == 1.0)  # top-1: the routed expert's weight is exactly 1
    zero = dict(inp)
    zero["w2"] = torch.zeros_like(inp["w2"])
    r0 = orc.layer_shared(zero, sh, w.K, w.W, w.cf)
    np.testing.assert_array_equal(r0["out"], r0["shared_y"])


@pytest.mark.parametrize("seed", range(8))
def test_slot_major_priority_brute_force(orc, seed):
    """Slot-major priority (every token's first choice before any second choice,
    [MoE 推理服务工程真相 2026, §4.3: which assignments give way when an expert is full]):
    positions, rows and the packed order against an O(N*K*E) recount."""
    rng = np.random.default_rng(seed)
    N, E, K, W = 12, 6, 3, 3
    lg = rng.standard_normal((N, E)).astype(np.float32)
    lg[:, 0] += 1.5  # a hot expert, so capacity binds
    idx, _, _ = orc.topk(lg, K)
    for C in (1, 3, 5, N * K):
        p = orc.positions(idx, E, W, C, order=orc.SLOT_MAJOR)
        b = brute.dispatch(idx, E, W, C, order=1)
        for key in ("counts", "kept", "offsets", "row_of", "packed_row_of"):
            np.testing.assert_array_equal(p[key], b[key], err_msg=(C, key))
        np.testing.assert_array_equal(p["D"], b["D"])
        assert p["stats"]["dedup_pairs"] == b["dedup"]
        # the token-major and slot-major results agree when nothing is dropped
        if C == N * K:
            q = orc.positions(idx, E, W, C)
            np.testing.assert_array_equal(q["kept"], p["kept"])


def test_slot_major_keeps_first_choices(orc):
    """Under slot-major priority, when capacity allows every first choice, no first
    choice is dropped; token-major priority can drop a later token's first choice."""
    idx = np.array([[0, 1], [0, 1], [1, 0]], np.int32)  # 3 tokens, K = 2, E = 2
    C = 2
    tm = orc.positions(idx, 2, 1, C)
    sm = orc.positions(idx, 2, 1, C, order=orc.SLOT_MAJOR)
    # token-major: expert 1 is filled by tokens 0 and 1 (their second choices), so token 2's
    # first choice (expert 1) is dropped
    assert tm["row_of"].reshape(3, 2)[2, 0] == -1
    # slot-major: first choices (0, 0, 1) are placed before any second choice
    assert np.all(sm["row_of"].reshape(3, 2)[:, 0] >= 0)


def test_drop_policies_hand_worked_example(orc):
    """The four drop policies on a 4-token example worked by hand
    (tests/golden/reroute_example.json)."""
    with open(os.path.join(GOLDEN, "reroute_example.json"), encoding="utf-8") as fh:
        g = json.load(fh)
    lg = np.array(g["logits"], np.float32)
    idx, _, _ = orc.topk(lg, g["K"])
    np.testing.assert_array_equal(idx, g["topk_idx"])
    for name, c in g["cases"].items():
        p = orc.positions(idx, g["E"], g["W"], g["C"], order=c["order"], reroute=c["reroute"],
                          logits=lg)
        np.testing.assert_array_equal(p["expert_of"], c["expert_of"], err_msg=name)
        np.testing.assert_array_equal(p["row_of"], c["row_of"], err_msg=name)
        np.testing.assert_array_equal(p["kept"], c["kept"], err_msg=name)
        assert p["stats"]["dropped"] == c["dropped"] and p["stats"]["rerouted"] == c["rerouted"]
        if "D" in c:
            np.testing.assert_array_equal(p["D"], c["D"], err_msg=name)
            np.testing.assert_array_equal(p["packed_row_of"], c["packed_row_of"], err_msg=name)
            assert p["stats"]["cross_rows"] == c["cross_rows"]
            assert p["stats"]["dedup_pairs"] == c["dedup_pairs"]


@pytest.mark.parametrize("seed", range(10))
def test_reroute_brute_force(orc, seed):
    """Re-routing of overflowed assignments to the next-best non-full expert, both
    priority orders, against an independent O((N*K)^2) restatement."""
    rng = np.random.default_rng(100 + seed)
    W = int(rng.choice([1, 2, 3]))
    E = W * int(rng.integers(2, 5))
    K = int(rng.integers(1, min(E, 4) + 1))
    N = W * int(rng.integers(2, 9))
    lg = rng.standard_normal((N, E)).astype(np.float32)
    lg[:, : max(1, E // 3)] += 1.2  # a few hot experts
    if seed % 3 == 0:
        lg = np.round(lg * 2) / 2  # ties between candidates
    idx, _, _ = orc.topk(lg, K)
    for C in (1, 2, max(1, N * K // E)):
        for order in (0, 1):
            p = orc.positions(idx, E, W, C, order=order, reroute=True, logits=lg)
            b = brute.dispatch(idx, E, W, C, order=order, reroute=True, logits=lg)
            for key in ("counts", "kept", "offsets", "row_of", "packed_row_of", "expert_of"):
                np.testing.assert_array_equal(p[key], b[key], err_msg=(C, order, key))
            np.testing.assert_array_equal(p["D"], b["D"])
            assert p["stats"]["dedup_pairs"] == b["dedup"]
            assert p["stats"]["rerouted"] == b["rerouted"]
            # invariants: no expert above capacity, no token twice at one expert,
            # re-routing never drops more than the plain policy
            assert p["kept"].max(initial=0) <= C
            eo = p["expert_of"].reshape(N, K)
            for t in range(N):
                got = eo[t][eo[t] >= 0]
                assert len(set(got.tolist())) == len(got)
            plain = orc.positions(idx, E, W, C, order=order)
            assert p["stats"]["dropped"] == plain["stats"]["dropped"] - p["stats"]["rerouted"]


# --------------------------------------------------------------------------- FP8 payload
# e4m3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no infinities, 448 the largest.

E4M3_HAND = [  # (value, code): format corners and round-to-nearest-even ties, worked by hand
    (0.0, 0x00), (-0.0, 0x80), (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (-448.0, 0xFE),
    (500.0, 0x7E),  # saturates
    (2.0 ** -9, 0x01), (7 * 2.0 ** -9, 0x07), (2.0 ** -6, 0x08),  # subnormals, smallest normal
    (2.0 ** -10, 0x00),  # half the smallest subnormal: tie to the even code 0
    (3 * 2.0 ** -10, 0x02),  # 1.5 subnormal quanta: tie to 2
    (1.0625, 0x38),  # halfway 1.0 / 1.125: even mantissa 0
    (1.1875, 0x3A),  # halfway 1.125 / 1.25: even mantissa 2
    (240.0, 0x77), (256.0, 0x78), (416.0, 0x7D), (432.0, 0x7E),  # 432 halfway 416 / 448 -> 448
]


def test_e4m3_hand_values(orc):
    v = np.array([a for a, _ in E4M3_HAND])
    np.testing.assert_array_equal(orc.e4m3_encode(v), [c for _, c in E4M3_HAND])
    assert np.isnan(orc.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()
    assert orc.e4m3_encode(np.array([np.nan]))[0] == 0x7F


def test_e4m3_round_trip_every_code(orc):
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    np.testing.assert_array_equal(orc.e4m3_encode(orc.e4m3_decode(codes)), codes)
    vals = orc.e4m3_decode(codes[codes < 0x80])
    assert np.all(np.diff(vals) > 0) and vals.max() == 448.0  # monotone codes, largest 448


def test_e4m3_matches_torch_float8(orc):
    """torch's float8_e4m3fn conversion is an independent implementation of the same
    rounding: agree on random values and on every tie."""
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(100000) * 30,
                        rng.uniform(-448, 448, 50000),
                        np.exp(rng.uniform(-16, 6, 50000)) * rng.choice([-1, 1], 50000)])
    codes = np.arange(0x7F, dtype=np.uint8)
    grid = orc.e4m3_decode(codes[codes != 0x7F])
    v = np.concatenate([v, (grid[1:] + grid[:-1]) / 2, -(grid[1:] + grid[:-1]) / 2])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(orc.e4m3_encode(v), ref)


def test_e4m3_scale_exponent(orc):
    assert orc.e4m3_scale_exponent(0.0) == 0
    assert orc.e4m3_scale_exponent(448.0) == 0 and orc.e4m3_scale_exponent(449.0) == 1
    assert orc.e4m3_scale_exponent(1.0) == -8  # 1 * 2^8 = 256 <= 448 < 512
    assert orc.e4m3_scale_exponent(float("inf")) == 0
    rng = np.random.default_rng(1)
    for amax in np.exp(rng.uniform(-80, 80, 2000)):
        j = orc.e4m3_scale_exponent(amax)
        assert 224.0 < math.ldexp(amax, -j) <= 448.0  # the smallest power of two that fits


def test_quantize_rows(orc):
    """Row quantisation = per-row power-of-two scale + e4m3 rounding, checked against
    torch's float8 conversion of the scaled rows; the scaled row maximum lies in (224, 448],
    so its code lies in [224, 448] (224.x may round down to 224)."""
    rng = np.random.default_rng(2)
    a = torch.from_numpy(rng.standard_normal((64, 96)) * np.exp(rng.uniform(-20, 20, (64, 1))))
    a = a.to(torch.bfloat16)
    a[3] = 0.0
    codes, scale = orc.quantize_rows_e4m3(a)
    af = a.double().numpy()
    for r in range(a.shape[0]):
        j = orc.e4m3_scale_exponent(np.abs(af[r]).max())
        assert scale[r] == math.ldexp(1.0, j)
        ref = torch.from_numpy(af[r] / scale[r]).to(torch.float8_e4m3fn).view(torch.uint8)
        np.testing.assert_array_equal(codes[r], ref.numpy())
        if r != 3:
            assert 224.0 <= np.abs(orc.e4m3_decode(codes[r])).max() <= 448.0
    assert np.all(codes[3] == 0) and scale[3] == 1.0
    # dequantised values are exact bf16 and within half an e4m3 step of the input
    deq = orc.dequantize_rows_bf16(codes, scale)
    back = (deq.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rel = np.abs(back - af) / np.maximum(np.abs(af), 2.0 ** -6 * scale[:, None])
    assert rel.max() <= 2.0 ** -4


def test_quantize_blocks_is_the_row_rule_per_block(orc):
    """Block quantisation of the return payload = the (pinned) row quantisation applied to
    each 32-column block as a row of its own, on bf16-representable values; and the same
    rule checked directly against torch's float8 conversion on fp32 values."""
    rng = np.random.default_rng(5)
    a = torch.from_numpy(rng.standard_normal((24, 128)) *
                         np.exp(rng.uniform(-30, 30, (24, 4))).repeat(32, axis=1))
    a = a.to(torch.bfloat16)
    a[2, 32:64] = 0.0
    codes, exps = orc.quantize_blocks_e4m3(a.double().numpy())
    rc, rs = orc.quantize_rows_e4m3(a.reshape(-1, 32))
    np.testing.assert_array_equal(codes.reshape(-1, 32), rc)
    np.testing.assert_array_equal(np.ldexp(1.0, exps.reshape(-1)), rs.astype(np.float64))
    assert exps[2, 1] == 0 and np.all(codes[2, 32:64] == 0)
    # fp32 values (not bf16): torch's conversion of each block scaled by 2^-j
    v = (rng.standard_normal((16, 96)) * np.exp(rng.uniform(-10, 10, (16, 3))).repeat(32, axis=1)
         ).astype(np.float32).astype(np.float64)
    codes, exps = orc.quantize_blocks_e4m3(v)
    for b in range(3):
        blk = v[:, 32 * b:32 * b + 32]
        for r in range(16):
            j = orc.e4m3_scale_exponent(np.abs(blk[r]).max())
            assert exps[r, b] == j
            ref = torch.from_numpy(np.ldexp(blk[r], -j)).to(torch.float8_e4m3fn).view(torch.uint8)
            np.testing.assert_array_equal(codes[r, 32 * b:32 * b + 32], ref.numpy())
    back = orc.dequantize_blocks_e4m3(codes, exps)
    floor = np.ldexp(2.0 ** -6, np.repeat(exps, 32, axis=1))   # below: e4m3 subnormals
    assert (np.abs(back - v) / np.maximum(np.abs(v), floor)).max() <= 2.0 ** -4


def test_quantize_blocks_hand_values(orc):
    """One row, two blocks: block 0 has largest magnitude 448 (j = 0: the codes are the values'
    own e4m3 codes), block 1 has 449 (j = 1: every value halved first)."""
    row = np.zeros((1, 64))
    row[0, 0], row[0, 1], row[0, 2] = 448.0, -1.0, 0.3
    row[0, 32], row[0, 33] = 449.0, 3.0
    codes, exps = orc.quantize_blocks_e4m3(row)
    assert exps.tolist() == [[0, 1]]
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0xB8   # 448; -1.0 = sign, exponent 7
    assert orc.e4m3_decode(codes[0, 2:3])[0] == 0.3125    # 0.3 -> nearest e4m3 (0.3125)
    assert orc.e4m3_decode(codes[0, 32:34]).tolist() == [224.0, 1.5]  # 224.5 -> 224; 1.5


def test_layer_fp8_reduces_to_bf16_layer_on_e4m3_inputs(orc):
    """With x, W1, W3, W2 already e4m3 values whose rows reach the top binade, quantising
    them is the identity: the FP8 layer's h equals the bf16 layer's h exactly, and its
    expert outputs differ only by h's roundings (to bf16, then to e4m3: within
    (2^-4 + 2^-8) relative per element), element by element within
    (2^-4 + 2^-8 + 2^-40) * sum_j |W2_ij h_j|; on ordinary inputs the output stays within the
    FP8 bar (three mantissa bits per operand: <= 2^-4 relative per element; bar 0.1)."""
    w = WORKLOADS["tiny"]
    inp = make_layer_inputs(w, seed=3)
    rng = np.random.default_rng(3)
    grid = orc.e4m3_decode(np.arange(0x7F, dtype=np.uint8))

    def e4m3_like(shape, scale_exp):
        v = rng.choice(grid[1:], size=shape) * rng.choice([-1.0, 1.0], size=shape)
        v[..., 0] = 448.0  # every row's maximum in the top binade: scale exactly 2^scale_exp
        return torch.from_numpy(v * 2.0 ** scale_exp).to(torch.bfloat16)

    exact = dict(inp, x=e4m3_like(tuple(inp["x"].shape), -12),
                 w1=e4m3_like(tuple(inp["w1"].shape), -14),
                 w3=e4m3_like(tuple(inp["w3"].shape), -14),
                 w2=e4m3_like(tuple(inp["w2"].shape), -14))
    a = orc.layer_fp8(exact, w.K, w.W, w.cf, want_h=True)
    b = orc.layer(exact, w.K, w.W, w.cf, want_h=True)
    assert np.all(a["fp8"]["sx"] == 2.0 ** -12) and np.all(a["fp8"]["s1"] == 2.0 ** -14)
    assert np.all(a["fp8"]["s2"] == 2.0 ** -14)
    np.testing.assert_array_equal(a["h_rows"], b["h_rows"])
    w2 = exact["w2"].double().numpy()
    row_expert = a["expert_of"][a["assign_of_row"]]
    mag = np.stack([np.abs(w2[e]) @ np.abs(a["h_rows"][i]) for i, e in enumerate(row_expert)])
    assert np.all(np.abs(a["y_rows"] - b["y_rows"]) <= (2.0 ** -4 + 2.0 ** -8 + 2.0 ** -40) * mag)
    assert np.abs(a["y_rows"] - b["y_rows"]).max() > 0  # h really was rounded
    r8 = orc.layer_fp8(inp, w.K, w.W, w.cf)
    r16 = orc.layer(inp, w.K, w.W, w.cf)
    np.testing.assert_array_equal(r8["row_of"], r16["row_of"])  # routing is on the bf16 x
    dev = np.linalg.norm(r8["out"] - r16["out"]) / np.linalg.norm(r16["out"])
    assert 1e-3 < dev <= 0.1, dev


BF16_HAND = [  # (value, bits), worked by hand: 1 sign, 8 exponent, 7 mantissa bits
    (1.0, 0x3F80), (-2.0, 0xC000), (0.0, 0x0000), (-0.0, 0x8000),
    (1.0 + 2.0 ** -8, 0x3F80),  # halfway 1 / 1 + 2^-7: even mantissa 0
    (1.0 + 3 * 2.0 ** -8, 0x3F82),  # halfway 1 + 2^-7 / 1 + 2^-6: even mantissa 2
    (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81),  # just above halfway
    ((2.0 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),  # largest finite
    ((2.0 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),  # halfway to 2^128: even -> infinity
    (2.0 ** -133, 0x0001), (2.0 ** -134, 0x0000), (3 * 2.0 ** -134, 0x0002),  # subnormals
]


def test_round_bf16_hand_values_and_exact_nearest(orc):
    v = np.array([a for a, _ in BF16_HAND])
    np.testing.assert_array_equal(orc.round_bf16(v), [b for _, b in BF16_HAND])
    # random doubles: the result is the nearer of the two bf16 neighbours (exact rationals),
    # ties to the even code
    from fractions import Fraction
    rng = np.random.default_rng(9)
    vals = rng.standard_normal(3000) * np.exp(rng.uniform(-30, 30, 3000))
    got = orc.round_bf16(vals)
    for x, b in zip(vals, got):
        g = float(np.array([int(b) << 16], np.uint32).view(np.float32)[0])
        lo_bits = int(np.array([g], np.float32).view(np.uint32)[0]) >> 16
        nb = [((lo_bits + s) & 0xFFFF) for s in (-1, 1)]
        for n in nb:
            o = float(np.array([n << 16], np.uint32).view(np.float32)[0])
            if np.isfinite(o) and np.sign(o) == np.sign(g):
                dg, do = abs(Fraction(g) - Fraction(x)), abs(Fraction(o) - Fraction(x))
                assert dg < do or (dg == do and (int(b) & 1) == 0), (x, hex(int(b)), hex(n))
    # float32-exact inputs: torch's float32 -> bf16 rounding is a second implementation
    f32 = (rng.standard_normal(20000) * 50).astype(np.float32)
    ref = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(orc.round_bf16(f32.astype(np.float64)), ref)


def test_down_rows_matches_matmul(orc):
    rng = np.random.default_rng(10)
    E, d, f, n = 3, 24, 40, 17
    w2 = torch.from_numpy(rng.standard_normal((E, d, f)) * 0.1).to(torch.bfloat16)
    h = torch.from_numpy(rng.standard_normal((n, f))).to(torch.bfloat16)
    re = rng.integers(0, E, n).astype(np.int32)
    y = orc.down_rows(re, orc.as_u16(h), w2)
    ref = np.stack([w2[e].double().numpy() @ h[i].double().numpy() for i, e in enumerate(re)])
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_layer_fp8_down_noise_bounded(orc):
    """The all-FP8 expert path (e4m3 x, W1, W3, then e4m3 h and W2) against the bf16 layer:
    routing identical, deviation of the output above zero and within the FP8 bar 0.1; the
    e4m3 h rows dequantise to within 2^-4 of the bf16 h."""
    w = WORKLOADS["tiny"]
    inp = make_layer_inputs(w, seed=4)
    r8 = orc.layer_fp8(inp, w.K, w.W, w.cf)
    r16 = orc.layer(inp, w.K, w.W, w.cf)
    np.testing.assert_array_equal(r8["row_of"], r16["row_of"])
    dev = np.linalg.norm(r8["out"] - r16["out"]) / np.linalg.norm(r16["out"])
    assert 1e-3 < dev <= 0.1, dev
    q = r8["fp8"]
    hb = (q["h_bf16"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    hd = (orc.dequantize_rows_bf16(q["hq"], q["hs"]).astype(np.uint32) << 16).view(
        np.float32).astype(np.float64)
    rel = np.abs(hd - hb) / np.maximum(np.abs(hb), 2.0 ** -6 * q["hs"][:, None])
    assert rel.max() <= 2.0 ** -4


# --------------------------------------------------------------------------- fp16 y payload
# fp16: 1 sign, 5 exponent bits (bias 15), 10 mantissa bits, largest finite 65504.

F16_HAND = [  # (value, bits): format corners and round-to-nearest-even ties, worked by hand
    (0.0, 0x0000), (-0.0, 0x8000), (1.0, 0x3C00), (-2.0, 0xC000), (65504.0, 0x7BFF),
    (65520.0, 0x7C00),  # halfway 65504 / 65536: ties to the even, out of range -> infinity
    (65519.0, 0x7BFF),
    (2.0 ** -24, 0x0001), (2.0 ** -14, 0x0400), (1023 * 2.0 ** -24, 0x03FF),  # subnormals
    (2.0 ** -25, 0x0000),  # half the smallest subnormal: ties to the even code 0
    (3 * 2.0 ** -25, 0x0002),  # 1.5 quanta: ties to 2
    (1.0 + 2.0 ** -11, 0x3C00),  # halfway 1 / 1 + 2^-10: even mantissa 0
    (1.0 + 3 * 2.0 ** -11, 0x3C02),  # halfway 1 + 2^-10 / 1 + 2^-9: even mantissa 2
    (1.0 / 3.0, 0x3555),
]


def test_f16_hand_values(orc):
    v = np.array([a for a, _ in F16_HAND])
    np.testing.assert_array_equal(orc.round_f16(v), [c for _, c in F16_HAND])
    assert orc.round_f16(np.array([np.nan]))[0] & 0x7C00 == 0x7C00


def test_f16_matches_torch_float16(orc):
    """torch's float32 -> float16 conversion is an independent implementation of the same
    rounding: agree on random fp32 values over the whole range and on every tie of a binade.
    (From float64 torch rounds twice, through float32, and differs at near-ties: 155.9374935
    lies below the 155.9375 tie and is 155.875, torch gives 156; the payload's values are
    fp32, where one rounding is the definition.)"""
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(100000) * 100,
                        np.exp(rng.uniform(-20, 11.2, 100000)) * rng.choice([-1, 1], 100000)])
    grid = np.arange(0x3C00, 0x4000, dtype=np.uint16).view(np.float16).astype(np.float64)
    v = np.concatenate([v, (grid[1:] + grid[:-1]) / 2, -(grid[1:] + grid[:-1]) / 2])
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(orc.round_f16(v32.astype(np.float64)), ref)
    assert orc.round_f16(np.array([155.93749352322445]))[0] == 0x58DF  # below the tie


def test_f16_scale_exponent(orc):
    assert orc.f16_scale_exponent(0.0) == 0 and orc.f16_scale_exponent(float("nan")) == 0
    assert orc.f16_scale_exponent(65504.0) == 0 and orc.f16_scale_exponent(65505.0) == 1
    assert orc.f16_scale_exponent(1.0) == -15  # 2^15 = 32768 <= 65504 < 65536
    rng = np.random.default_rng(8)
    for amax in np.exp(rng.uniform(-60, 60, 2000)):
        j = orc.f16_scale_exponent(amax)
        assert 32752.0 < math.ldexp(amax, -j) <= 65504.0  # the smallest power of two that fits
    assert orc.f16_scale_exponent(1e-40) == -126  # clamped: the exponent byte stays in range


def test_quantize_blocks_f16(orc):
    """Each 32-column block: exponent from its largest magnitude by the rule above, codes =
    torch's float16 conversion of the block scaled by 2^-j; dequantised values within half an
    fp16 step of the input (relative 2^-11 of the block's scale-adjusted top binade)."""
    rng = np.random.default_rng(9)
    v = (rng.standard_normal((20, 128)) * np.exp(rng.uniform(-40, 40, (20, 4))).repeat(32, axis=1)
         ).astype(np.float32).astype(np.float64)
    v[4, 64:96] = 0.0
    codes, exps = orc.quantize_blocks_f16(v)
    for b in range(4):
        blk = v[:, 32 * b:32 * b + 32]
        for r in range(20):
            j = orc.f16_scale_exponent(np.abs(blk[r]).max())
            assert exps[r, b] == j
            ref = torch.from_numpy(np.ldexp(blk[r], -j)).to(torch.float16)
            np.testing.assert_array_equal(codes[r, 32 * b:32 * b + 32],
                                          ref.view(torch.int16).numpy().view(np.uint16))
    assert exps[4, 2] == 0 and np.all(codes[4, 64:96] == 0)
    back = orc.dequantize_blocks_f16(codes, exps)
    scale = np.exp2(np.repeat(exps, 32, axis=1).astype(np.float64))
    assert np.all(np.abs(back - v) <= 2.0 ** -11 * np.maximum(np.abs(v), 2.0 ** -14 * scale))
