"""Parity of the CUDA path (through the C ABI) with the CPU oracle on shapes the
oracle finishes in seconds: several tiles per expert, ragged tails, drops,
empty experts, K = E, E = 1. Integer outputs bit-exact; floating-point outputs
within relative Frobenius 5e-3 and max-abs 2e-2 * RMS of the oracle, on every case,
and within the per-element bound the arithmetic implies."""
import numpy as np
import pytest
import torch

from layer_runner import (assert_rounded_h, assert_within_bound, assert_within_tolerance,
                          h_bound_rows, run_layer, run_stages, tolerance_report)
from moe_workloads import WORKLOADS, Workload, make_layer_inputs

pytestmark = pytest.mark.gpu

CASES = [
    WORKLOADS["tiny"],
    # ~260 rows per expert: 3 M-tiles with a ragged last tile; G2 with 256-wide N tiles
    Workload("ragged", N=1040, d=256, f=384, E=8, K=2, W=4),
    # capacity drops under Zipf skew; d = 384 takes the 128-wide N tile of G2
    Workload("drop_bn128", N=384, d=384, f=256, E=6, K=3, W=3, cf=1.25, s=1.1),
    # many experts with few rows, some with none; heavy Zipf skew with drops gives a
    # heavy-tailed output (a few elements near 7x its RMS): the case where a bf16 h would
    # miss the max-abs bar (2.1% of the RMS) and the fp16 h meets it (0.3%)
    Workload("sparse_experts", N=256, d=128, f=128, E=64, K=6, W=8, cf=1.0, s=1.2),
    Workload("k_eq_e", N=64, d=128, f=128, E=4, K=4, W=2),
    Workload("dense_e1", N=300, d=256, f=256, E=1, K=1, W=1),
    Workload("decode_like", N=16, d=512, f=256, E=64, K=8, W=8),
    Workload("odd_e", N=100, d=128, f=128, E=5, K=2, W=5, cf=0.9),
    Workload("one_token_per_rank", N=8, d=128, f=128, E=16, K=3, W=8, cf=0.5),
    Workload("wide_k", N=96, d=128, f=128, E=48, K=32, W=4),
    # every limit at once, token-major: 256 experts, K = 32, 64 ranks, capacity drops
    Workload("max_limits", N=128, d=128, f=128, E=256, K=32, W=64, cf=1.0),
    # >= 768 rows per expert on average: the CTA-pair GEMM kernel (256-row tiles)
    Workload("pair_tiles", N=1600, d=256, f=256, E=2, K=1, W=2),
    # skewed rows (Zipf bias): large experts on the pair kernel, small ones on the
    # single-CTA kernel, in the same GEMM
    Workload("pair_split", N=3200, d=256, f=256, E=4, K=1, W=4, s=1.6),
    # slot-major drop priority (first choices before second choices)
    Workload("slot_major_drop", N=384, d=384, f=256, E=6, K=3, W=3, cf=1.0, s=1.1,
             slot_major=True),
    Workload("slot_major_ragged", N=1040, d=256, f=384, E=8, K=2, W=4, cf=0.8, s=0.8,
             slot_major=True),
    Workload("slot_major_wide_k", N=96, d=128, f=128, E=48, K=32, W=4, cf=0.75, s=1.0,
             slot_major=True),
    # 256 experts, K = 32, 64 ranks: the scan's 2048 segment starts per expert live in
    # global memory instead of shared memory (no Zipf skew: with it, most assignments drop
    # and the output tail alone takes bf16 rounding of h to the max-abs bar)
    Workload("slot_major_many_segments", N=128, d=128, f=128, E=256, K=32, W=64, cf=1.0,
             slot_major=True),
    Workload("slot_major_dropless", N=200, d=128, f=128, E=10, K=3, W=5, slot_major=True),
    # overflowed assignments re-routed to the next-best non-full expert
    Workload("reroute_drop", N=384, d=384, f=256, E=6, K=3, W=3, cf=1.0, s=1.1, reroute=True),
    Workload("reroute_slot_major", N=1040, d=256, f=384, E=8, K=2, W=4, cf=0.8, s=0.8,
             slot_major=True, reroute=True),
    Workload("reroute_many_experts", N=256, d=128, f=128, E=64, K=6, W=8, cf=1.0, s=0.6,
             reroute=True),
    # 256 experts: eight logits per lane in the ranking warp
    Workload("reroute_e256", N=128, d=128, f=128, E=256, K=8, W=8, cf=0.5, reroute=True),
    # K = E: every expert is routed to by every token, so there is no candidate
    Workload("reroute_all_full", N=64, d=128, f=128, E=4, K=4, W=2, cf=0.5, reroute=True),
]


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_float_outputs(ref, got, inp, w, stated_bar: bool = True):
    """h, y and out against the oracle: per element within the bound the arithmetic implies
    (one rounding of h in the precision the run stored it in, fp32 accumulation), relative
    Frobenius 5e-3, and, when `stated_bar`, max-abs 2e-2 * RMS on y and on the output."""
    R = ref["R"]
    assert_rounded_h(got["h"][:R], ref["h_rows"], "h", w.d)
    row_expert = ref["expert_of"][ref["assign_of_row"]]
    ybound = h_bound_rows(ref["h_rows"], inp["w2"], got.get("w2_used"), row_expert)
    assert_within_bound(got["y"][:R], ref["y_rows"], ybound, "y")
    obound = np.zeros((w.N, w.d))
    for a in np.nonzero(ref["row_of"] >= 0)[0]:
        wa = abs(float(ref["topk_w"].reshape(-1)[a]))
        r = ref["row_of"][a]
        # propagated y bound, plus the fp32 weights and the fp32 sum over K slots
        obound[a // w.K] += wa * ybound[r] + (w.K + 8) * 2.0 ** -24 * wa * np.abs(ref["y_rows"][r])
    assert_within_bound(got["out"], ref["out"], obound, "out")
    if stated_bar:
        assert_within_tolerance(got["y"][:R], ref["y_rows"], "y")
        return assert_within_tolerance(got["out"], ref["out"], "out")
    rep = tolerance_report(got["out"], ref["out"])
    assert rep["rel_frob"] <= 5e-3, rep
    return rep


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("seed", [0, 1])
def test_layer_stages_match_oracle(orc, w, seed):
    inp = make_layer_inputs(w, seed=seed)
    ref = orc.layer(inp, w.K, w.W, w.cf, want_h=True, order=int(w.slot_major),
                    reroute=w.reroute)
    got = run_stages(inp, w)
    assert got["dev_error"] == 0

    # a1: logits bit for bit; a2: selection exact, weights to fp32 rounding
    np.testing.assert_array_equal(got["logits"].cpu().numpy().view(np.uint32),
                                  ref["logits"].view(np.uint32))
    np.testing.assert_array_equal(got["topk_idx"].cpu().numpy(), ref["topk_idx"])
    np.testing.assert_allclose(got["topk_w"].cpu().numpy(), ref["topk_w"], rtol=2e-6, atol=1e-7)

    # a3: integer bookkeeping, bit-exact
    R = ref["R"]
    for key, rk in (("counts", "counts"), ("kept", "kept"), ("offsets", "offsets"),
                    ("row_of", "row_of")):
        np.testing.assert_array_equal(got[key].cpu().numpy(), ref[rk], err_msg=key)
    assign = got["assign"].cpu().numpy()
    np.testing.assert_array_equal(assign[:R], ref["assign_of_row"])
    assert np.all(assign[R:] == -7), "rows past R must not be written"
    np.testing.assert_array_equal(got["D"].cpu().numpy().reshape(w.W, w.W), ref["D"])
    np.testing.assert_array_equal(got["pk_off"].cpu().numpy(), ref["pk_off"])
    st, rs = got["stats"], ref["stats"]
    assert (st["rows"], st["dropped"], st["cross_rows"], st["dedup_pairs"]) == (
        rs["R"], rs["dropped"], rs["cross_rows"], rs["dedup_pairs"])
    assert (st["active_experts"], st["max_kept"], st["min_kept"]) == (
        rs["active_experts"], rs["max_kept"], rs["min_kept"])
    assert st["rerouted"] == rs["rerouted"]
    if w.reroute:
        np.testing.assert_array_equal(got["expert_of"].cpu().numpy(), ref["expert_of"])
    assert st["capacity"] == min(ref["C"], w.N * w.K)

    # a4: scatter is an exact copy, in both layouts
    xu = _u16(inp["x"])
    np.testing.assert_array_equal(_u16(got["x_sorted"][:R]), xu[ref["assign_of_row"] // w.K])
    kept_slots = np.nonzero(ref["row_of"] >= 0)[0]
    packed = np.empty((R, w.d), np.uint16)
    packed[ref["packed_row_of"][kept_slots]] = xu[kept_slots // w.K]
    np.testing.assert_array_equal(_u16(got["x_packed"][:R]), packed)

    # a5/a6: expert GEMMs; a7: combine (fp16 h: the stated bar on every case)
    check_float_outputs(ref, got, inp, w)

    # the fused entry point runs the same kernels: identical bits
    lay = run_layer(inp, w)
    assert lay["dev_error"] == 0
    np.testing.assert_array_equal(lay["out"].cpu().numpy().view(np.uint32),
                                  got["out"].cpu().numpy().view(np.uint32))
    np.testing.assert_array_equal(lay["topk_idx"].cpu().numpy(), ref["topk_idx"])
    assert lay["stats"]["dedup_pairs"] == rs["dedup_pairs"]


BF16_H_CASES = ["tiny", "ragged", "drop_bn128", "sparse_experts", "pair_split", "max_limits"]


@pytest.mark.parametrize("name", BF16_H_CASES)
def test_layer_bf16_h_mode(orc, name):
    """The bf16 precision of h (MOE_FLAG_H_BF16; W2 in bf16): every output within the
    per-element bound of one bf16 rounding of h and the relative Frobenius bar. The max-abs bar
    is not claimed for this mode: on a heavy-tailed output (sparse_experts) one bf16 rounding
    of h moves the largest element by about 2 % of the output's RMS."""
    w = next(c for c in CASES if c.name == name)
    inp = make_layer_inputs(w, seed=0)
    ref = orc.layer(inp, w.K, w.W, w.cf, want_h=True, order=int(w.slot_major),
                    reroute=w.reroute)
    got = run_stages(inp, w, h_bf16=True)
    assert got["dev_error"] == 0
    assert got["h"].dtype == torch.bfloat16
    np.testing.assert_array_equal(got["row_of"].cpu().numpy(), ref["row_of"])
    rep = check_float_outputs(ref, got, inp, w, stated_bar=False)
    lay = run_layer(inp, w, h_bf16=True)
    np.testing.assert_array_equal(lay["out"].cpu().numpy().view(np.uint32),
                                  got["out"].cpu().numpy().view(np.uint32))
    print(name, "bf16 h", rep)


def test_convert_bf16_to_f16_matches_torch():
    """The fp16 copy of the weights: bit for bit torch's own bf16 -> fp16 conversion (round to
    nearest even), and the count of changed elements equal to the count of values that are
    not fp16 numbers, on N(0, 0.02) weights plus hand-picked corners (tiny, subnormal in fp16,
    the largest finite fp16, beyond it)."""
    import combine_grouped_gemm_router_b200 as m
    g = torch.Generator().manual_seed(3)
    w = (torch.randn(1 << 20, generator=g) * 0.02).to(torch.bfloat16)
    corners = torch.tensor([0.0, -0.0, 2.0 ** -17, -2.0 ** -18, 3.0 * 2.0 ** -20, 2.0 ** -24,
                            2.0 ** -26, 1e-30, 65504.0, -65504.0, 1.0, -448.0, 3.0e38, -7e4,
                            2.0 ** -14, 0.5], dtype=torch.float32).to(torch.bfloat16)
    src = torch.cat([w, corners]).cuda()
    dst = torch.empty(src.shape, dtype=torch.float16, device="cuda")
    changed = torch.zeros(1, dtype=torch.int64, device="cuda")
    m.moe_convert_bf16_to_f16(src, dst, changed)
    torch.cuda.synchronize()
    ref = src.cpu().to(torch.float16)
    assert torch.equal(dst.cpu().view(torch.int16), ref.view(torch.int16))
    n_changed = int((ref.float() != src.cpu().float()).sum())
    assert int(changed.item()) == n_changed and n_changed > 0
    # the two values beyond 65504 became infinite: recorded in the device error word
    assert m.moe_get_device_error(True) == 9
    assert m.moe_get_device_error(True) == 0


def test_residual_combine(orc):
    w = Workload("res", N=128, d=256, f=256, E=8, K=2, W=4, cf=1.0)
    inp = make_layer_inputs(w, seed=5)
    ref = orc.layer(inp, w.K, w.W, w.cf)
    import combine_grouped_gemm_router_b200 as m
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf)
    dev = torch.device("cuda")
    ws = torch.empty(m.moe_layer_workspace_size(shape), dtype=torch.uint8, device=dev)
    x = inp["x"].to(dev)
    out = torch.empty(w.N, w.d, dtype=torch.float32, device=dev)
    w2 = m.w2_for(shape, inp["w2"].to(dev))
    m.moe_layer(shape, x, inp["w_router"].to(dev), None, inp["w1"].to(dev), inp["w3"].to(dev),
                w2, out, residual=x, ws=ws)
    # bf16 output mode (the next layer's input), out of place
    shape16 = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf, out_bf16=True)
    out16 = torch.empty(w.N, w.d, dtype=torch.bfloat16, device=dev)
    m.moe_layer(shape16, x, inp["w_router"].to(dev), None, inp["w1"].to(dev), inp["w3"].to(dev),
                w2, out16, residual=x, ws=ws)
    torch.cuda.synchronize()
    xr = inp["x"].double().numpy()
    assert_within_tolerance(out, xr + ref["out"], "x + moe(x)")
    # the bf16 output is the fp32 output rounded once
    assert torch.equal(out16, out.to(torch.bfloat16))


def test_identity_experts_round_trip():
    """Dispatch then combine with y := x_sorted returns x * sum of kept weights."""
    import combine_grouped_gemm_router_b200 as m
    w = Workload("id", N=512, d=256, f=128, E=16, K=4, W=4)
    inp = make_layer_inputs(w, seed=3)
    got = run_stages(inp, w)
    shape = got["shape"]
    out = torch.empty(w.N, w.d, dtype=torch.float32, device="cuda")
    m.moe_combine(shape, got["x_sorted"].float(), got["row_of"], got["topk_w"], out)
    torch.cuda.synchronize()
    wsum = got["topk_w"].double().sum(1, keepdim=True).cpu().numpy()
    assert np.allclose(wsum, 1.0, atol=1e-6)
    assert_within_tolerance(out, inp["x"].double().numpy() * wsum, "identity round trip")


def test_affinity_kernel_matches_oracle(orc):
    rng = np.random.default_rng(0)
    N, E, K = 5000, 64, 6
    a, _, _ = orc.topk(rng.standard_normal((N, E)).astype(np.float32), K)
    b, _, _ = orc.topk(rng.standard_normal((N, E)).astype(np.float32), K)
    import combine_grouped_gemm_router_b200 as m
    cnt = torch.zeros(E, E, dtype=torch.int64, device="cuda")
    m.moe_affinity_accumulate(N, E, K, torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), cnt)
    m.moe_affinity_accumulate(N, E, K, torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), cnt)
    ref = orc.affinity(a, b, E)
    np.testing.assert_array_equal(cnt.cpu().numpy(), 2 * ref)
    # the global-atomic path (E > 64)
    E2 = 96
    a2, _, _ = orc.topk(rng.standard_normal((N, E2)).astype(np.float32), K)
    b2, _, _ = orc.topk(rng.standard_normal((N, E2)).astype(np.float32), K)
    cnt2 = torch.zeros(E2, E2, dtype=torch.int64, device="cuda")
    m.moe_affinity_accumulate(N, E2, K, torch.from_numpy(a2).cuda(), torch.from_numpy(b2).cuda(),
                              cnt2)
    np.testing.assert_array_equal(cnt2.cpu().numpy(), orc.affinity(a2, b2, E2))
    assert m.moe_get_device_error(True) == 0


def test_residual_moe_layer(orc):
    """Residual-MoE: routed experts plus a shared dense MLP on every token, summed in the
    combine. moe_shared_expert against the oracle's dense MLP; moe_layer_shared against the
    oracle's layer and, bit for bit, against the same stages called one by one."""
    import combine_grouped_gemm_router_b200 as m
    from moe_workloads import make_shared_inputs
    for w in (Workload("res_small", N=256, d=256, f=256, E=4, K=1, W=2, shared_f=384),
              Workload("res_k2_drop", N=300, d=384, f=128, E=6, K=2, W=3, cf=1.0, s=1.1,
                       shared_f=128)):
        inp = make_layer_inputs(w, seed=1)
        sh = make_shared_inputs(w, seed=1)
        ref = orc.layer_shared(inp, sh, w.K, w.W, w.cf)
        dev = torch.device("cuda")
        shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf)
        shd = {k: v.to(dev) for k, v in sh.items()}
        shd["ws2"] = m.w2_for(shape, shd["ws2"])  # the down projection's weights in fp16
        h_s = torch.empty(w.N, w.shared_f, dtype=torch.float16, device=dev)
        y_s = torch.empty(w.N, w.d, dtype=torch.float32, device=dev)
        ws_s = torch.empty(256, dtype=torch.uint8, device=dev)
        x = inp["x"].to(dev)
        m.moe_shared_expert(shape, w.shared_f, x, shd["ws1"], shd["ws3"], shd["ws2"], h_s, y_s, ws_s)
        torch.cuda.synchronize()
        assert_within_tolerance(y_s, ref["shared_y"], "shared MLP")
        got = run_stages(inp, w)
        out_st = torch.empty(w.N, w.d, dtype=torch.float32, device=dev)
        m.moe_combine(shape, got["y"], got["row_of"], got["topk_w"], out_st, shared_y=y_s)
        ws = torch.empty(m.moe_layer_shared_workspace_size(shape, w.shared_f), dtype=torch.uint8,
                         device=dev)
        out = torch.empty(w.N, w.d, dtype=torch.float32, device=dev)
        bias = None if inp["bias"] is None else inp["bias"].to(dev)
        m.moe_layer_shared(shape, w.shared_f, x, inp["w_router"].to(dev), bias, inp["w1"].to(dev),
                           inp["w3"].to(dev), got["w2_used"], shd["ws1"], shd["ws3"], shd["ws2"],
                           out, ws=ws)
        torch.cuda.synchronize()
        assert m.moe_get_device_error(True) == 0
        assert torch.equal(out, out_st)
        assert_within_tolerance(out, ref["out"], w.name)


@pytest.mark.parametrize("d", [8, 24])
@pytest.mark.parametrize("slot_major", [False, True])
def test_route_dispatch_small_hidden(orc, d, slot_major):
    """Routing and dispatch at the smallest hidden sizes the boundary accepts (d % 8 == 0;
    the GEMMs need d % 128): logits, selection, bookkeeping and both scatter layouts, exact."""
    w = Workload(f"small_d{d}", N=96, d=d, f=128, E=6, K=2, W=3, cf=1.0, s=1.0,
                 slot_major=slot_major)
    inp = make_layer_inputs(w, seed=4)
    ref = orc.route_and_dispatch(inp["x"], inp["w_router"], inp["bias"], w.K, w.W, w.cf,
                                 order=int(slot_major))
    got = run_stages(inp, w)
    assert got["dev_error"] == 0 and "h" not in got
    np.testing.assert_array_equal(got["logits"].cpu().numpy().view(np.uint32),
                                  ref["logits"].view(np.uint32))
    np.testing.assert_array_equal(got["topk_idx"].cpu().numpy(), ref["topk_idx"])
    for key in ("counts", "kept", "offsets", "row_of"):
        np.testing.assert_array_equal(got[key].cpu().numpy(), ref[key], err_msg=key)
    R = ref["R"]
    xu = _u16(inp["x"])
    np.testing.assert_array_equal(_u16(got["x_sorted"][:R]), xu[ref["assign_of_row"] // w.K])
    kept_slots = np.nonzero(ref["row_of"] >= 0)[0]
    packed = np.empty((R, w.d), np.uint16)
    packed[ref["packed_row_of"][kept_slots]] = xu[kept_slots // w.K]
    np.testing.assert_array_equal(_u16(got["x_packed"][:R]), packed)
    np.testing.assert_array_equal(got["D"].cpu().numpy().reshape(w.W, w.W), ref["D"])


@pytest.mark.parametrize("scale", [1.0, 400.0])
def test_fp16_range_pass(orc, scale):
    """Activations beyond fp16's range (x scaled by 400: |h| far above 65504): the range pass
    stores h * 2^-k and the down projection multiplies back by 2^k, so the layer stays within
    the stated bar of the oracle and no error is recorded; in range (scale 1) the record stays
    below 65504 and the second pass does nothing."""
    import combine_grouped_gemm_router_b200 as m
    w = Workload("range", N=256, d=256, f=256, E=8, K=2, W=4)
    inp = make_layer_inputs(w, seed=6)
    inp["x"] = (inp["x"].float() * scale).to(torch.bfloat16)
    ref = orc.layer(inp, w.K, w.W, w.cf, want_h=True)
    got = run_stages(inp, w)
    assert got["dev_error"] == 0
    R = ref["R"]
    amax = got["h"][-1].view(torch.int32)[0:2].cpu().numpy().view(np.uint32)[0]
    top = float(np.abs(ref["h_rows"]).max())
    assert np.float32(amax.view(np.float32)) == pytest.approx(top, rel=2e-3)
    assert (top > 65504) == (scale > 1)
    if scale > 1:  # h was stored scaled into range: compare it scaled back
        k = int(np.ceil(np.log2(top / 65504.0)))
        hk = got["h"][:R].double() * 2.0 ** k
        rel = float(((hk.cpu().numpy() - ref["h_rows"]) ** 2).sum() / (ref["h_rows"] ** 2).sum())
        assert rel ** 0.5 <= 5e-3
    assert_within_tolerance(got["y"][:R], ref["y_rows"], "y")
    assert_within_tolerance(got["out"], ref["out"], "out")
    lay = run_layer(inp, w)
    assert lay["dev_error"] == 0
    assert torch.equal(lay["out"], got["out"])
