"""Parity at the full workload sizes, in the launch configuration the bench times.

Inputs are drawn on the GPU with a seeded generator and copied to the host for
the oracle. Routing, counts, positions, the mapping table, the traffic matrix,
the pack offsets and the counters are compared in full, bit for bit; both
scatter layouts are checked row for row; expert outputs and the layer output
are checked on a sample of tokens (first, last and seeded-random ones) that the
oracle computes one by one, against the stated tolerance."""
import numpy as np
import pytest
import torch

from layer_runner import (assert_within_bound, assert_within_tolerance, bf16_h_bound_rows,
                          run_stages, tolerance_report)
from moe_workloads import STACK_GRID_CF, STACK_GRID_S, WORKLOADS, make_layer_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def sample_tokens(N: int, n: int = 24, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, N - 1), size=min(n - 2, max(N - 2, 0)), replace=False) \
        if N > 2 else np.array([], dtype=np.int64)
    return np.unique(np.concatenate([[0, N - 1], mid])).astype(np.int64)


def host_inputs(inp: dict, experts=None) -> dict:
    """Copy to the host what the oracle needs; with `experts`, only those experts'
    weights, renumbered 0..len-1 (the caller renumbers its expert ids alike)."""
    out = {"x": inp["x"].cpu(), "w_router": inp["w_router"].cpu(),
           "bias": None if inp["bias"] is None else inp["bias"].cpu()}
    for k in ("w1", "w3", "w2"):
        out[k] = inp[k][experts].cpu() if experts is not None else inp[k].cpu()
    return out


def check_full_size(orc, w, seed=0, n_sample=24):
    torch.cuda.empty_cache()
    inp = make_layer_inputs(w, seed=seed, device="cuda")
    got = run_stages(inp, w)
    assert got["dev_error"] == 0
    hx = host_inputs(inp, experts=[])  # routing needs no expert weights
    r = orc.route_and_dispatch(hx["x"], hx["w_router"], hx["bias"], w.K, w.W, w.cf,
                               order=int(w.slot_major), reroute=w.reroute)

    # routing and bookkeeping, in full
    np.testing.assert_array_equal(got["logits"].cpu().numpy().view(np.uint32),
                                  r["logits"].view(np.uint32))
    np.testing.assert_array_equal(got["topk_idx"].cpu().numpy(), r["topk_idx"])
    np.testing.assert_allclose(got["topk_w"].cpu().numpy(), r["topk_w"], rtol=2e-6, atol=1e-7)
    for key in ("counts", "kept", "offsets", "row_of"):
        np.testing.assert_array_equal(got[key].cpu().numpy(), r[key], err_msg=key)
    R = r["R"]
    np.testing.assert_array_equal(got["assign"][:R].cpu().numpy(), r["assign_of_row"])
    np.testing.assert_array_equal(got["D"].cpu().numpy().reshape(w.W, w.W), r["D"])
    np.testing.assert_array_equal(got["pk_off"].cpu().numpy(), r["pk_off"])
    st, rs = got["stats"], r["stats"]
    assert (st["rows"], st["dropped"], st["cross_rows"], st["dedup_pairs"], st["active_experts"],
            st["max_kept"], st["min_kept"], st["rerouted"]) == (
                rs["R"], rs["dropped"], rs["cross_rows"], rs["dedup_pairs"], rs["active_experts"],
                rs["max_kept"], rs["min_kept"], rs["rerouted"])
    if w.reroute:
        np.testing.assert_array_equal(got["expert_of"].cpu().numpy(), r["expert_of"])

    # both scatter layouts, every row (indices verified above)
    aor = torch.from_numpy(r["assign_of_row"]).cuda().long()
    assert torch.equal(got["x_sorted"][:R], inp["x"][aor // w.K])
    kept_slots = torch.from_numpy(np.nonzero(r["row_of"] >= 0)[0]).cuda()
    prow = torch.from_numpy(r["packed_row_of"]).cuda().long()[kept_slots]
    assert torch.equal(got["x_packed"][prow], inp["x"][kept_slots // w.K])

    # sampled tokens through the experts: the oracle computes them one by one
    toks = sample_tokens(w.N, n_sample, seed)
    slots = (toks[:, None] * w.K + np.arange(w.K)[None, :]).reshape(-1)
    eo = r["expert_of"][slots]
    used = np.unique(eo[eo >= 0])
    remap = np.full(w.E, -1, np.int64)
    remap[used] = np.arange(len(used))
    hx = host_inputs(inp, experts=torch.from_numpy(used).cuda())
    rr = dict(r)
    # compact weight numbering for the experts the sampled rows use
    rr["expert_of"] = np.where(r["expert_of"] >= 0, remap[r["expert_of"]], -1).astype(np.int32)
    smp = orc.layer_sampled(hx, w.K, w.W, w.cf, toks, routing=rr, want_h=True)
    rows = torch.from_numpy(smp["sample_rows"]).cuda().long()
    rep_h = tolerance_report(got["h"][rows], smp["sample_h"])
    assert rep_h["rel_frob"] <= 5e-3, rep_h
    # y and out: the per-element bound of one bf16 rounding of h (the down projection's
    # operand) plus fp32 accumulation, and the relative Frobenius bar; the max-abs bar is
    # asserted when nothing is dropped and reported otherwise (with heavy drops many
    # sampled tokens have zero output, which deflates the RMS the bar is relative to)
    w2 = hx["w2"].double().numpy()
    sample_expert = rr["expert_of"][smp["sample_slots"]]
    ybound = bf16_h_bound_rows(smp["sample_h"], w2, sample_expert)
    assert_within_bound(got["y"][rows], smp["sample_y"], ybound, "y sample")
    obound = np.zeros_like(smp["out_tokens"])
    pos = {int(a): i for i, a in enumerate(smp["sample_slots"])}
    for li, t in enumerate(toks):
        for k in range(w.K):
            a = int(t) * w.K + k
            if a in pos:
                wa = abs(float(r["topk_w"].reshape(-1)[a]))
                yi = pos[a]
                obound[li] += wa * ybound[yi] + (w.K + 8) * 2.0 ** -24 * wa * np.abs(
                    smp["sample_y"][yi])
    got_out = got["out"][torch.from_numpy(toks).cuda()]
    assert_within_bound(got_out, smp["out_tokens"], obound, "out sample")
    rep_y = tolerance_report(got["y"][rows], smp["sample_y"])
    rep_o = tolerance_report(got_out, smp["out_tokens"])
    assert rep_y["rel_frob"] <= 5e-3 and rep_o["rel_frob"] <= 5e-3, (rep_y, rep_o)
    if r["stats"]["dropped"] == 0:
        assert_within_tolerance(got["y"][rows], smp["sample_y"], "y sample")
        assert_within_tolerance(got_out, smp["out_tokens"], "out sample")
    # routing margins (reported; the logits are bit-exact, so no seed is rejected)
    lg = np.sort(r["logits"], axis=1)[:, ::-1]
    margin = lg[:, w.K - 1] - lg[:, w.K] if w.K < w.E else np.full(w.N, np.inf)
    return dict(R=R, y=rep_y, out=rep_o, h=rep_h, min_margin=float(margin.min()),
                tokens_margin_below_1e5=int((margin < 1e-5).sum()))


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
@pytest.mark.parametrize("name", ["mixtral_prefill", "e128_skew", "decode"])
def test_full_size_workload(orc, name, seed):
    rep = check_full_size(orc, WORKLOADS[name], seed=seed)
    print(name, seed, rep)


@pytest.mark.parametrize("name", ["e128_skew", "stack4"])
def test_full_size_slot_major(orc, name):
    """Slot-major drop priority at full size, with capacity binding under the Zipf skew."""
    w = WORKLOADS[name].with_(slot_major=True, s=1.2, cf=1.0)
    rep = check_full_size(orc, w, n_sample=16)
    print(name, "slot-major", rep)


@pytest.mark.parametrize("slot_major", [False, True])
@pytest.mark.parametrize("name", ["e128_skew", "stack4"])
def test_full_size_reroute(orc, name, slot_major):
    """Re-routing of overflowed assignments at full size, capacity binding under the skew."""
    w = WORKLOADS[name].with_(reroute=True, slot_major=slot_major, s=1.2, cf=1.0)
    rep = check_full_size(orc, w, n_sample=16)
    print(name, "reroute", "slot-major" if slot_major else "token-major", rep)


@pytest.mark.parametrize("cf", STACK_GRID_CF)
@pytest.mark.parametrize("s", STACK_GRID_S)
def test_full_size_stack_layer(orc, cf, s):
    w = WORKLOADS["stack4"].with_(cf=cf, s=s)
    rep = check_full_size(orc, w, n_sample=16)
    print("stack4 layer 0", cf, s, rep)


def test_stack_affinity_full_size(orc):
    """The affinity counts of the 4-layer stack at full size (N=32768, E=64, K=6).

    Exactness of the count: each layer pair is counted by the GPU kernel from routing
    that the oracle produced for seeded inputs of those two layers, and compared bit
    for bit with the oracle's count. Then the stack itself runs on the GPU (each layer
    fed the previous layer's output x + MoE(x), rounded to bf16) and its affinity
    counts satisfy the invariants exactly: row sums are K times the tokens routed to
    the row's expert, the total is K^2 N, and they equal a recount of its own routing."""
    import combine_grouped_gemm_router_b200 as m
    w = WORKLOADS["stack4"].with_(cf=1.25, s=1.2)
    N, E, K = w.N, w.E, w.K
    routes = []
    for layer in range(2):
        inp = make_layer_inputs(w, seed=layer, device="cuda")
        hx = host_inputs(inp, experts=[])
        lg = orc.router_logits(hx["x"], hx["w_router"], hx["bias"])
        routes.append(orc.topk(lg, K)[0])
        del inp
    cnt = torch.zeros(E, E, dtype=torch.int64, device="cuda")
    m.moe_affinity_accumulate(N, E, K, torch.from_numpy(routes[0]).cuda(),
                              torch.from_numpy(routes[1]).cuda(), cnt)
    np.testing.assert_array_equal(cnt.cpu().numpy(), orc.affinity(routes[0], routes[1], E))

    # the stack on the GPU
    shape = m.make_shape(N, w.d, w.f, E, K, w.W, w.cf, out_bf16=True)
    ws = torch.empty(m.moe_layer_workspace_size(shape), dtype=torch.uint8, device="cuda")
    x = make_layer_inputs(w, seed=0, device="cuda")["x"]
    topks = []
    for layer in range(w.layers):
        lin = make_layer_inputs(w, seed=0, device="cuda", layer=layer, with_x=False)
        topk = torch.empty(N, K, dtype=torch.int32, device="cuda")
        nxt = torch.empty_like(x)
        m.moe_layer(shape, x, lin["w_router"], lin["bias"], lin["w1"], lin["w3"], lin["w2"], nxt,
                    residual=x, topk_idx_out=topk, ws=ws)
        topks.append(topk)
        x = nxt
        del lin
    torch.cuda.synchronize()
    assert m.moe_get_device_error(True) == 0
    for j in range(w.layers - 1):
        c = torch.zeros(E, E, dtype=torch.int64, device="cuda")
        m.moe_affinity_accumulate(N, E, K, topks[j], topks[j + 1], c)
        c = c.cpu().numpy()
        a = topks[j].cpu().numpy()
        b = topks[j + 1].cpu().numpy()
        n_i = np.bincount(a.reshape(-1), minlength=E)
        np.testing.assert_array_equal(c.sum(1), K * n_i)
        assert c.sum() == K * K * N
        recount = np.zeros((E, E), np.int64)
        np.add.at(recount, (np.repeat(a, K, axis=1).reshape(-1), np.tile(b, (1, K)).reshape(-1)), 1)
        np.testing.assert_array_equal(c, recount)
        P = c / np.maximum(n_i[:, None], 1)
        print(f"layer pair {j}->{j + 1}: max P(p|i) = {P.max():.3f}, diag mass "
              f"{np.trace(c) / c.sum():.4f}")


def test_full_size_residual_moe(orc):
    """Residual-MoE at the Mixtral shape with top-1 routing and a shared MLP of the same width:
    routing in full, the layer output on sampled tokens (routed part + shared MLP)."""
    import combine_grouped_gemm_router_b200 as m
    from moe_workloads import make_shared_inputs
    w = WORKLOADS["residual_top1"]
    torch.cuda.empty_cache()
    inp = make_layer_inputs(w, seed=0, device="cuda")
    sh = make_shared_inputs(w, seed=0, device="cuda")
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf)
    ws = torch.empty(m.moe_layer_shared_workspace_size(shape, w.shared_f), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(w.N, w.d, dtype=torch.float32, device="cuda")
    topk = torch.empty(w.N, w.K, dtype=torch.int32, device="cuda")
    m.moe_layer_shared(shape, w.shared_f, inp["x"], inp["w_router"], inp["bias"], inp["w1"],
                       inp["w3"], inp["w2"], sh["ws1"], sh["ws3"], sh["ws2"], out,
                       topk_idx_out=topk, ws=ws)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(True) == 0
    hx = host_inputs(inp, experts=[])
    r = orc.route_and_dispatch(hx["x"], hx["w_router"], hx["bias"], w.K, w.W, w.cf)
    np.testing.assert_array_equal(topk.cpu().numpy(), r["topk_idx"])
    toks = sample_tokens(w.N, 16, 0)
    slots = (toks[:, None] * w.K + np.arange(w.K)[None, :]).reshape(-1)
    eo = r["expert_of"][slots]
    used = np.unique(eo[eo >= 0])
    remap = np.full(w.E, -1, np.int64)
    remap[used] = np.arange(len(used))
    hx = host_inputs(inp, experts=torch.from_numpy(used).cuda())
    rr = dict(r)
    rr["expert_of"] = np.where(r["expert_of"] >= 0, remap[r["expert_of"]], -1).astype(np.int32)
    smp = orc.layer_sampled(hx, w.K, w.W, w.cf, toks, routing=rr)
    dense = orc.shared_expert(hx["x"][torch.from_numpy(toks)], sh["ws1"].cpu(), sh["ws3"].cpu(),
                              sh["ws2"].cpu())
    rep = assert_within_tolerance(out[torch.from_numpy(toks).cuda()], smp["out_tokens"] + dense,
                                  "residual-MoE sample")
    print("residual_top1", rep)
