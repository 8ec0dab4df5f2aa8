"""Parity at the full workload sizes, in the launch configuration the bench times.

Inputs are drawn on the GPU with a seeded generator and copied to the host for
the oracle. Routing, counts, positions, the mapping table, the traffic matrix,
the pack offsets and the counters are compared in full, bit for bit; both
scatter layouts are checked row for row; expert outputs and the layer output
are checked against the stated tolerance (relative Frobenius 5e-3, max-abs
2e-2 * RMS) on a sample of tokens (first, last and seeded-random ones) that the
oracle computes one by one, and on the whole output of the 128-expert, decode and
Mixtral-shaped layers. The stack of four layers is checked layer by layer with
the oracle fed the GPU's own input to each layer (teacher forcing): routing and
the inter-layer affinity counts bit for bit, each layer's output at the bar."""
import numpy as np
import pytest
import torch

from layer_runner import (assert_rounded_h, assert_within_bound, assert_within_tolerance,
                          decode_y_payload, f16_payload_bound, h_bound_rows, run_stages,
                          tolerance_report)
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


def check_full_size(orc, w, seed=0, n_sample=24, y_f16=False):
    """With y_f16 the expert outputs travel as the fp16 block payload: its decoded rows are
    checked against the oracle's y within the fp32 bound widened by the payload's rounding."""
    torch.cuda.empty_cache()
    inp = make_layer_inputs(w, seed=seed, device="cuda")
    got = run_stages(inp, w, y_f16=y_f16)
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
    assert_rounded_h(got["h"][rows], smp["sample_h"], "h sample", w.d)
    rep_h = tolerance_report(got["h"][rows], smp["sample_h"])
    # y and out: the per-element bound of one rounding of h (the down projection's operand,
    # fp16) plus fp32 accumulation, the relative Frobenius bar and the max-abs bar
    sample_expert = rr["expert_of"][smp["sample_slots"]]
    ybound = h_bound_rows(smp["sample_h"], hx["w2"], got["w2_used"][torch.from_numpy(used).cuda()],
                          sample_expert)
    y_got = got["y"][rows]
    if y_f16:
        y_got = decode_y_payload(got["shape"], got["y"], rows)
        ybound = f16_payload_bound(ybound, smp["sample_y"])
    assert_within_bound(y_got, smp["sample_y"], ybound, "y sample")
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
    rep_y = assert_within_tolerance(y_got, smp["sample_y"], "y sample")
    rep_o = assert_within_tolerance(got_out, smp["out_tokens"], "out sample")
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


@pytest.mark.parametrize("name", ["mixtral_prefill", "e128_skew", "decode", "stack4"])
def test_full_size_y_f16(orc, name):
    """The layers with the fp16 return payload (the bench's default for the non-FP8 path)."""
    rep = check_full_size(orc, WORKLOADS[name], y_f16=True)
    print(name, "y fp16 payload", rep)


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


def full_output_check(orc, w, seed=0, y_f16=False):
    """The whole output of one layer (every token, every column) against the oracle's layer
    computed in full: routing bit for bit, h within its rounding, y and the output per element
    within the bound the arithmetic implies and within the stated bar (with y_f16, y is the
    decoded fp16 block payload and its bound includes the payload's rounding)."""
    torch.cuda.empty_cache()
    inp = make_layer_inputs(w, seed=seed, device="cuda")
    got = run_stages(inp, w, y_f16=y_f16)
    assert got["dev_error"] == 0
    hx = host_inputs(inp)
    ref = orc.layer(hx, w.K, w.W, w.cf, want_h=True, order=int(w.slot_major), reroute=w.reroute)
    np.testing.assert_array_equal(got["topk_idx"].cpu().numpy(), ref["topk_idx"])
    np.testing.assert_array_equal(got["row_of"].cpu().numpy(), ref["row_of"])
    R = ref["R"]
    assert_rounded_h(got["h"][:R], ref["h_rows"], "h", w.d)
    row_expert = ref["expert_of"][ref["assign_of_row"]]
    ybound = h_bound_rows(ref["h_rows"], hx["w2"], got["w2_used"].cpu(), row_expert)
    y_got = got["y"][:R]
    if y_f16:
        y_got = decode_y_payload(got["shape"], got["y"], torch.arange(R, device="cuda"))
        ybound = f16_payload_bound(ybound, ref["y_rows"])
    assert_within_bound(y_got, ref["y_rows"], ybound, "y")
    kept = np.nonzero(ref["row_of"] >= 0)[0]
    wa = np.abs(ref["topk_w"].reshape(-1)[kept].astype(np.float64))[:, None]
    rows = ref["row_of"][kept]
    per_slot = wa * ybound[rows] + (w.K + 8) * 2.0 ** -24 * wa * np.abs(ref["y_rows"][rows])
    obound = np.zeros((w.N, w.d))
    np.add.at(obound, kept // w.K, per_slot)
    assert_within_bound(got["out"], ref["out"], obound + 1e-30, "out")
    rep_y = assert_within_tolerance(y_got, ref["y_rows"], "y")
    rep_o = assert_within_tolerance(got["out"], ref["out"], "out")
    return dict(R=R, dropped=ref["stats"]["dropped"], y=rep_y, out=rep_o)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_full_output_e128_skew(orc, seed):
    """The 128-expert layer with Zipf skew and capacity drops (two thirds of the assignments
    dropped): every element of the output, four seeds."""
    rep = full_output_check(orc, WORKLOADS["e128_skew"], seed)
    assert rep["dropped"] > 0
    print("e128_skew full output", seed, rep)


@pytest.mark.parametrize("name", ["e128_skew", "decode"])
def test_full_output_y_f16(orc, name):
    """Every element of the 128-expert and decode layers with the fp16 return payload."""
    rep = full_output_check(orc, WORKLOADS[name], 0, y_f16=True)
    print(name, "full output, y fp16 payload", rep)


def test_full_output_decode(orc):
    rep = full_output_check(orc, WORKLOADS["decode"], 0)
    print("decode full output", rep)


def test_full_output_mixtral_prefill(orc):
    """The Mixtral-shaped layer in full: 2.9 TFLOP for the oracle (about a minute on 16 host
    cores)."""
    rep = full_output_check(orc, WORKLOADS["mixtral_prefill"], 0)
    print("mixtral_prefill full output", rep)


def sampled_output_check(orc, inp, w, r, toks, got_out, w2_used, y_f16=False):
    """The layer output of the tokens `toks` (got_out, fp32 rows in the order of toks) against
    the oracle's expert FFN and combine of those tokens under the routing r: per element within
    the propagated bound (with y_f16, widened by the fp16 payload's rounding), and the stated
    bar."""
    slots = (toks[:, None] * w.K + np.arange(w.K)[None, :]).reshape(-1)
    eo = r["expert_of"][slots]
    used = np.unique(eo[eo >= 0])
    remap = np.full(w.E, -1, np.int64)
    remap[used] = np.arange(len(used))
    ut = torch.from_numpy(used).to(inp["w1"].device)
    hx = host_inputs(inp, experts=ut)
    rr = dict(r)
    rr["expert_of"] = np.where(r["expert_of"] >= 0, remap[r["expert_of"]], -1).astype(np.int32)
    smp = orc.layer_sampled(hx, w.K, w.W, w.cf, toks, routing=rr, want_h=True)
    sample_expert = rr["expert_of"][smp["sample_slots"]]
    ybound = h_bound_rows(smp["sample_h"], hx["w2"], w2_used[ut].cpu(), sample_expert)
    if y_f16:
        ybound = f16_payload_bound(ybound, smp["sample_y"])
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
    assert_within_bound(got_out, smp["out_tokens"], obound, "out sample")
    return assert_within_tolerance(got_out, smp["out_tokens"], "out sample")


def stack_teacher_forced(orc, w, n_sample=16, y_f16=False):
    """The stack of w.layers layers on the GPU, x_{j+1} = bf16(x_j + MoE_j(x_j)), checked layer by
    layer against the oracle fed the GPU's own x_j (teacher forcing, so that the routing
    contract holds per layer):
     * the stack's step equals the layer's fp32 output plus x_j, rounded once to bf16;
     * topk_idx and the dispatch counters of layer j equal the oracle's on x_j, bit for bit;
     * the output of layer j on sampled tokens is within the stated bar of the oracle's;
     * the inter-layer affinity counts moe_affinity_accumulate forms from the GPU's routing
       equal the oracle's counts from its own routing, bit for bit.
    With y_f16 the layers pass their expert outputs to the combine as the fp16 block payload."""
    import combine_grouped_gemm_router_b200 as m
    N, d, E, K = w.N, w.d, w.E, w.K
    torch.cuda.empty_cache()
    shape32 = m.make_shape(N, d, w.f, E, K, w.W, w.cf, y_f16=y_f16)
    shape16 = m.make_shape(N, d, w.f, E, K, w.W, w.cf, out_bf16=True, y_f16=y_f16)
    ws = torch.empty(m.moe_layer_workspace_size(shape16), dtype=torch.uint8, device="cuda")
    x = make_layer_inputs(w, seed=0, device="cuda", with_x=True)["x"]
    gpu_routes, orc_routes, reports = [], [], []
    for layer in range(w.layers):
        lin = make_layer_inputs(w, seed=0, device="cuda", layer=layer, with_x=False)
        w2h = m.w2_for(shape32, lin["w2"])
        moe = torch.empty(N, d, dtype=torch.float32, device="cuda")
        topk = torch.empty(N, K, dtype=torch.int32, device="cuda")
        stats = m.stats_buffer()
        m.moe_layer(shape32, x, lin["w_router"], lin["bias"], lin["w1"], lin["w3"], w2h, moe,
                    topk_idx_out=topk, stats=stats, ws=ws)
        nxt = torch.empty_like(x)
        topk2 = torch.empty_like(topk)
        m.moe_layer(shape16, x, lin["w_router"], lin["bias"], lin["w1"], lin["w3"], w2h, nxt,
                    residual=x, topk_idx_out=topk2, ws=ws)
        torch.cuda.synchronize()
        assert m.moe_get_device_error(True) == 0
        assert torch.equal(topk, topk2)
        assert torch.equal(nxt, (moe + x.float()).to(torch.bfloat16)), "stack step"
        inp = dict(lin, x=x)
        hx = host_inputs(inp, experts=[])
        r = orc.route_and_dispatch(hx["x"], hx["w_router"], hx["bias"], K, w.W, w.cf)
        np.testing.assert_array_equal(topk.cpu().numpy(), r["topk_idx"])
        st, rs = m.stats_dict(m.read_stats(stats)), r["stats"]
        assert (st["rows"], st["dropped"], st["cross_rows"], st["dedup_pairs"],
                st["active_experts"], st["max_kept"], st["min_kept"]) == (
                    rs["R"], rs["dropped"], rs["cross_rows"], rs["dedup_pairs"],
                    rs["active_experts"], rs["max_kept"], rs["min_kept"])
        toks = sample_tokens(N, n_sample, seed=layer)
        rep = sampled_output_check(orc, inp, w, r, toks, moe[torch.from_numpy(toks).cuda()], w2h,
                                   y_f16=y_f16)
        reports.append(dict(layer=layer, dropped=rs["dropped"], **rep))
        gpu_routes.append(topk)
        orc_routes.append(r["topk_idx"])
        del lin, w2h
        x = nxt
    for j in range(w.layers - 1):
        c = torch.zeros(E, E, dtype=torch.int64, device="cuda")
        m.moe_affinity_accumulate(N, E, K, gpu_routes[j], gpu_routes[j + 1], c)
        ref = orc.affinity(orc_routes[j], orc_routes[j + 1], E)
        np.testing.assert_array_equal(c.cpu().numpy(), ref)
        assert int(ref.sum()) == K * K * N
    return reports


@pytest.mark.parametrize("cf", STACK_GRID_CF)
@pytest.mark.parametrize("s", STACK_GRID_S)
def test_stack_teacher_forced(orc, cf, s):
    """The 4-layer stack (N=32768, d=4096, f=1536, E=64, K=6) at every capacity factor and Zipf
    skew of its grid, each layer against the oracle on the GPU's own input."""
    reps = stack_teacher_forced(orc, WORKLOADS["stack4"].with_(cf=cf, s=s))
    print("stack4", cf, s, reps)


def test_stack_teacher_forced_y_f16(orc):
    """The stack as the bench runs it (capacity factor 1.25, no skew) with the fp16 return
    payload between each layer's down projection and combine."""
    reps = stack_teacher_forced(orc, WORKLOADS["stack4"], y_f16=True)
    print("stack4 y fp16 payload", reps)


def test_stack_teacher_forced_planted_affinity(orc):
    """The stack whose routers carry planted inter-layer affinity: the affinity counts (sparse,
    concentrated rows) bit for bit against the oracle's."""
    reps = stack_teacher_forced(orc, WORKLOADS["stack4_affinity"], n_sample=8)
    print("stack4_affinity", reps)


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
    w2h, ws2h = m.w2_for(shape, inp["w2"]), m.w2_for(shape, sh["ws2"])
    ws = torch.empty(m.moe_layer_shared_workspace_size(shape, w.shared_f), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(w.N, w.d, dtype=torch.float32, device="cuda")
    topk = torch.empty(w.N, w.K, dtype=torch.int32, device="cuda")
    m.moe_layer_shared(shape, w.shared_f, inp["x"], inp["w_router"], inp["bias"], inp["w1"],
                       inp["w3"], w2h, sh["ws1"], sh["ws3"], ws2h, out,
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
