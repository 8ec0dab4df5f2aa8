"""Parity of the FP8 payload path (e4m3 rows with per-row power-of-two scales, e4m3 gate/up
GEMM) with the oracle: quantisation codes and scales bit for bit, the bookkeeping bit for bit,
h within one bf16 rounding of the oracle's FP8 layer, y and the output within the derived bound
and the stated bar against the oracle's FP8 layer. Against the bf16 layer the FP8 path differs
by its quantisation noise; the bar for that is relative Frobenius <= 0.1 (three mantissa bits
on x and on W1, W3: <= 2^-4 relative error per element)."""
import numpy as np
import pytest
import torch

from layer_runner import (assert_rounded_bf16, assert_within_bound, assert_within_tolerance,
                          bf16_h_bound_rows, lib, tolerance_report)
from moe_workloads import WORKLOADS, Workload, make_layer_inputs

pytestmark = pytest.mark.gpu

FP8_VS_BF16_REL_FROB = 0.1


def _u8(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint8)


def quantize_weights(m, w):
    """e4m3 rows of W1 and W3 (per output channel) on the GPU."""
    E, f, d = w.shape
    q = torch.empty(E, f, d, dtype=torch.uint8, device=w.device)
    sc = torch.empty(E, f, dtype=torch.float32, device=w.device)
    m.moe_quantize_rows_e4m3(w, q, sc)
    return q, sc


def run_fp8_stages(inp, w, dev="cuda"):
    m = lib()
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf, slot_major=w.slot_major)
    N, K, E, W, d, f = w.N, w.K, w.E, w.W, w.d, w.f
    RA = m.moe_rows_alloc(shape)
    ws = torch.empty(m.moe_workspace_size(shape), dtype=torch.uint8, device=dev)
    x = inp["x"].to(dev)
    topk_idx = torch.empty(N, K, dtype=torch.int32, device=dev)
    topk_w = torch.empty(N, K, dtype=torch.float32, device=dev)
    m.moe_route(shape, x, inp["w_router"].to(dev),
                None if inp["bias"] is None else inp["bias"].to(dev), topk_idx, topk_w, None, ws)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    kept = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty(N * K, dtype=torch.int32, device=dev)
    assign = torch.full((RA,), -7, dtype=torch.int32, device=dev)
    xs = torch.zeros(RA, d, dtype=torch.uint8, device=dev)
    xp = torch.zeros(RA, d, dtype=torch.uint8, device=dev)
    ss = torch.zeros(RA, dtype=torch.float32, device=dev)
    ps = torch.zeros(RA, dtype=torch.float32, device=dev)
    stats = m.stats_buffer(dev)
    m.moe_dispatch_fp8(shape, x, topk_idx, counts, kept, offsets, row_of, assign, xs, ss,
                       x_packed=xp, packed_scale=ps, stats=stats, ws=ws)
    w1q, s1 = quantize_weights(m, inp["w1"].to(dev))
    w3q, s3 = quantize_weights(m, inp["w3"].to(dev))
    h = torch.zeros(RA, f, dtype=torch.bfloat16, device=dev)
    y = torch.zeros(RA, d, dtype=torch.float32, device=dev)
    m.moe_expert_up_fp8(shape, xs, ss, offsets, w1q, s1, w3q, s3, h)
    w2 = inp["w2"].to(dev)
    m.moe_expert_down(shape, h, offsets, w2, y)
    out = torch.empty(N, d, dtype=torch.float32, device=dev)
    m.moe_combine(shape, y, row_of, topk_w, out)
    # the fused entry point
    wsl = torch.empty(m.moe_layer_workspace_size(shape), dtype=torch.uint8, device=dev)
    out_l = torch.empty(N, d, dtype=torch.float32, device=dev)
    m.moe_layer_fp8(shape, x, inp["w_router"].to(dev),
                    None if inp["bias"] is None else inp["bias"].to(dev), w1q, s1, w3q, s3, w2,
                    out_l, ws=wsl)
    torch.cuda.synchronize()
    return dict(topk_idx=topk_idx, topk_w=topk_w, counts=counts, kept=kept, offsets=offsets,
                row_of=row_of, assign=assign, x_sorted=xs, x_packed=xp, sorted_scale=ss,
                packed_scale=ps, w1q=w1q, s1=s1, w3q=w3q, s3=s3, h=h, y=y, out=out,
                out_layer=out_l, stats=m.stats_dict(m.read_stats(stats)),
                dev_error=m.moe_get_device_error(True))


def test_quantize_rows_matches_oracle(orc):
    """Codes and scales bit for bit on rows of very different magnitudes, with zero rows
    and many exact ties (bf16 has 5 more mantissa bits than e4m3)."""
    m = lib()
    g = torch.Generator().manual_seed(5)
    a = torch.randn(300, 512, generator=g) * torch.exp(torch.randn(300, 1, generator=g) * 8)
    a = a.to(torch.bfloat16)
    a[7] = 0.0
    a[11, :] = 448.0
    a[12, 3] = -1e-30  # a tiny row maximum
    a[12, 4:] = 0.0
    codes = torch.empty(300, 512, dtype=torch.uint8, device="cuda")
    scale = torch.empty(300, dtype=torch.float32, device="cuda")
    m.moe_quantize_rows_e4m3(a.cuda(), codes, scale)
    torch.cuda.synchronize()
    rc, rs = orc.quantize_rows_e4m3(a)
    np.testing.assert_array_equal(_u8(codes), rc)
    np.testing.assert_array_equal(scale.cpu().numpy(), rs)


CASES = [
    Workload("fp8_small", N=64, d=128, f=256, E=8, K=2, W=4),
    # ragged tails and drops; d = 384 puts the single-CTA kernel on 3 atoms of 128
    Workload("fp8_drop", N=384, d=384, f=256, E=6, K=3, W=3, cf=1.25, s=1.1),
    # >= 768 rows per expert and d % 256 == 0: the CTA-pair kernel
    Workload("fp8_pair", N=1600, d=512, f=256, E=2, K=1, W=2),
    # skewed: pair tiles for the large experts, single-CTA tiles for the rest
    Workload("fp8_pair_split", N=3200, d=256, f=256, E=4, K=1, W=4, s=1.6),
    Workload("fp8_many_experts_slot_major", N=256, d=256, f=128, E=64, K=6, W=8, cf=1.0, s=0.6,
             slot_major=True),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("seed", [0, 1])
def test_fp8_layer_matches_oracle(orc, w, seed):
    inp = make_layer_inputs(w, seed=seed)
    ref = orc.layer_fp8(inp, w.K, w.W, w.cf, want_h=True, order=int(w.slot_major))
    got = run_fp8_stages(inp, w)
    assert got["dev_error"] == 0
    q = ref["fp8"]
    # weights: codes and scales bit for bit
    np.testing.assert_array_equal(_u8(got["w1q"]), q["w1q"])
    np.testing.assert_array_equal(got["s1"].cpu().numpy(), q["s1"])
    np.testing.assert_array_equal(_u8(got["w3q"]), q["w3q"])
    np.testing.assert_array_equal(got["s3"].cpu().numpy(), q["s3"])
    # bookkeeping as in the bf16 dispatch
    R = ref["R"]
    np.testing.assert_array_equal(got["topk_idx"].cpu().numpy(), ref["topk_idx"])
    for key in ("counts", "kept", "offsets", "row_of"):
        np.testing.assert_array_equal(got[key].cpu().numpy(), ref[key], err_msg=key)
    np.testing.assert_array_equal(got["assign"].cpu().numpy()[:R], ref["assign_of_row"])
    assert got["stats"]["dedup_pairs"] == ref["stats"]["dedup_pairs"]
    # the FP8 payload: every kept row's codes and scale, in both layouts
    tok = ref["assign_of_row"] // w.K
    np.testing.assert_array_equal(_u8(got["x_sorted"])[:R], q["xq"][tok])
    np.testing.assert_array_equal(got["sorted_scale"].cpu().numpy()[:R], q["sx"][tok])
    kept_slots = np.nonzero(ref["row_of"] >= 0)[0]
    prow = ref["packed_row_of"][kept_slots]
    np.testing.assert_array_equal(_u8(got["x_packed"])[prow], q["xq"][kept_slots // w.K])
    np.testing.assert_array_equal(got["packed_scale"].cpu().numpy()[prow],
                                  q["sx"][kept_slots // w.K])
    # h: one bf16 rounding of the oracle's FP8 gate/up; y and out: the derived bound
    assert_rounded_bf16(got["h"][:R], ref["h_rows"], "h")
    w2 = inp["w2"].double().numpy()
    ybound = bf16_h_bound_rows(ref["h_rows"], w2, ref["expert_of"][ref["assign_of_row"]])
    assert_within_bound(got["y"][:R], ref["y_rows"], ybound, "y")
    assert_within_tolerance(got["y"][:R], ref["y_rows"], "y")
    assert_within_tolerance(got["out"], ref["out"], "out")
    np.testing.assert_array_equal(got["out_layer"].cpu().numpy().view(np.uint32),
                                  got["out"].cpu().numpy().view(np.uint32))
    # the quantisation noise against the bf16 layer
    r16 = orc.layer(inp, w.K, w.W, w.cf, order=int(w.slot_major))
    dev = tolerance_report(got["out"], r16["out"])
    assert dev["rel_frob"] <= FP8_VS_BF16_REL_FROB, dev
    print(w.name, "fp8 vs bf16 layer", dev)


def test_fp8_layer_full_size_mixtral(orc):
    """The Mixtral-shaped layer (N=4096, d=4096, f=14336, E=8, K=2) through moe_layer_fp8:
    routing in full, the output on sampled tokens against the oracle's FP8 layer, whose
    operands are quantised on the host from the same bf16 inputs."""
    from test_gpu_fullsize import host_inputs, sample_tokens
    m = lib()
    w = WORKLOADS["mixtral_prefill"]
    torch.cuda.empty_cache()
    inp = make_layer_inputs(w, seed=0, device="cuda")
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf)
    w1q, s1 = quantize_weights(m, inp["w1"])
    w3q, s3 = quantize_weights(m, inp["w3"])
    ws = torch.empty(m.moe_layer_workspace_size(shape), dtype=torch.uint8, device="cuda")
    out = torch.empty(w.N, w.d, dtype=torch.float32, device="cuda")
    topk = torch.empty(w.N, w.K, dtype=torch.int32, device="cuda")
    m.moe_layer_fp8(shape, inp["x"], inp["w_router"], inp["bias"], w1q, s1, w3q, s3, inp["w2"],
                    out, topk_idx_out=topk, ws=ws)
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
    # the GPU's weight codes must equal the oracle's quantisation of the same rows
    q1, sc1 = orc.quantize_rows_e4m3(hx["w1"])
    np.testing.assert_array_equal(_u8(w1q[torch.from_numpy(used).cuda()]), q1)
    np.testing.assert_array_equal(s1[torch.from_numpy(used).cuda()].cpu().numpy(), sc1)
    q3, sc3 = orc.quantize_rows_e4m3(hx["w3"])
    xq, sx = orc.quantize_rows_e4m3(hx["x"])
    deq = dict(hx, x=torch.from_numpy(orc.dequantize_rows_bf16(xq, sx).view(np.int16)).view(
        torch.bfloat16), w1=torch.from_numpy(orc.dequantize_rows_bf16(q1, sc1).view(np.int16)).view(
        torch.bfloat16), w3=torch.from_numpy(orc.dequantize_rows_bf16(q3, sc3).view(np.int16)).view(
        torch.bfloat16))
    rr = dict(r)
    rr["expert_of"] = np.where(r["expert_of"] >= 0, remap[r["expert_of"]], -1).astype(np.int32)
    smp = orc.layer_sampled(deq, w.K, w.W, w.cf, toks, routing=rr)
    rep = assert_within_tolerance(out[torch.from_numpy(toks).cuda()], smp["out_tokens"],
                                  "fp8 layer sample")
    smp16 = orc.layer_sampled(hx, w.K, w.W, w.cf, toks, routing=rr)
    dev = tolerance_report(out[torch.from_numpy(toks).cuda()], smp16["out_tokens"])
    assert dev["rel_frob"] <= FP8_VS_BF16_REL_FROB, dev
    print("mixtral fp8", rep, "vs bf16", dev)
