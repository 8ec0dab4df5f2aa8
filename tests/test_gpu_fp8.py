"""Parity of the FP8 path (e4m3 dispatch rows with per-row power-of-two scales, e4m3 gate/up
and down GEMMs) with the oracle: quantisation codes and scales bit for bit, the bookkeeping bit
for bit, h within one bf16 rounding of the oracle's FP8 layer, the down GEMM on the oracle's own
e4m3 rows within fp32 accumulation error, and the layer output within a derived per-element
bound and the stated relative-Frobenius bar against the oracle's FP8 layer. Against the bf16
layer the FP8 path differs by its quantisation noise; the bar for that is relative Frobenius
<= 0.1 (three mantissa bits per operand: <= 2^-4 relative error per element).

h is computed in fp32 on the GPU and in fp64 by the oracle; both round it to bf16, and about one
element in 10^5 lands on the other side of a bf16 rounding boundary. Requantising such an
element to e4m3 can move its code by one step, which moves single outputs by up to one e4m3
step of one term: the per-element bound below includes exactly those steps."""
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
    """e4m3 rows of an expert weight tensor [E][rows][cols] (per output channel) on the GPU."""
    E, r, c = w.shape
    q = torch.empty(E, r, c, dtype=torch.uint8, device=w.device)
    sc = torch.empty(E, r, dtype=torch.float32, device=w.device)
    m.moe_quantize_rows_e4m3(w, q, sc)
    return q, sc


def deq(codes, scale, orc):
    """Dequantised e4m3 rows as float64."""
    return orc.e4m3_decode(codes) * np.asarray(scale, np.float64)[..., None]


def run_fp8_stages(inp, w, dev="cuda", fp8_return=False):
    m = lib()
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf, slot_major=w.slot_major,
                         fp8_return=fp8_return)
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
    w2q, s2 = quantize_weights(m, inp["w2"].to(dev))
    h = torch.zeros(RA, f, dtype=torch.bfloat16, device=dev)
    hq = torch.zeros(RA, f, dtype=torch.uint8, device=dev)
    hs = torch.zeros(RA, dtype=torch.float32, device=dev)
    y = (torch.zeros(m.moe_y_bytes(shape), dtype=torch.uint8, device=dev) if fp8_return
         else torch.zeros(RA, d, dtype=torch.float32, device=dev))
    m.moe_expert_up_fp8(shape, xs, ss, offsets, w1q, s1, w3q, s3, h)
    m.moe_quantize_rows_e4m3(h, hq, hs, rows_dev=offsets[E:])  # the kept rows of h
    m.moe_expert_down_fp8(shape, hq, hs, offsets, w2q, s2, y)
    out = torch.empty(N, d, dtype=torch.float32, device=dev)
    m.moe_combine(shape, y, row_of, topk_w, out)
    # the fused entry point
    wsl = torch.empty(m.moe_layer_workspace_size(shape), dtype=torch.uint8, device=dev)
    out_l = torch.empty(N, d, dtype=torch.float32, device=dev)
    m.moe_layer_fp8(shape, x, inp["w_router"].to(dev),
                    None if inp["bias"] is None else inp["bias"].to(dev), w1q, s1, w3q, s3, w2q, s2,
                    out_l, ws=wsl)
    torch.cuda.synchronize()
    return dict(topk_idx=topk_idx, topk_w=topk_w, counts=counts, kept=kept, offsets=offsets,
                row_of=row_of, assign=assign, x_sorted=xs, x_packed=xp, sorted_scale=ss,
                packed_scale=ps, w1q=w1q, s1=s1, w3q=w3q, s3=s3, w2q=w2q, s2=s2, h=h, hq=hq,
                hs=hs, y=y, out=out,
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
    np.testing.assert_array_equal(_u8(got["w2q"]), q["w2q"])
    np.testing.assert_array_equal(got["s2"].cpu().numpy(), q["s2"])
    # h: one bf16 rounding of the oracle's FP8 gate/up
    assert_rounded_bf16(got["h"][:R], ref["h_rows"], "h")
    # e4m3 rows of h: the oracle's codes, except one step where the two bf16 h differ
    hb_gpu = got["h"][:R].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    hq_gpu = _u8(got["hq"])[:R]
    hs_gpu = got["hs"].cpu().numpy()[:R]
    moved = hq_gpu != q["hq"]
    rows_scale_moved = hs_gpu != q["hs"]  # a row maximum crossed a power of two
    assert np.all((hb_gpu != q["h_bf16"]).any(axis=1)[rows_scale_moved])
    lone = moved & ~rows_scale_moved[:, None]
    assert np.all(hb_gpu[lone] != q["h_bf16"][lone]), "code moved without cause"
    assert moved.mean() <= 1e-3, moved.mean()
    dh = np.abs(deq(hq_gpu, hs_gpu, orc) - deq(q["hq"], q["hs"], orc))
    # y: |dy| <= sum_j |dh_j| |W2_ij| (code steps) + fp32 accumulation of sum_j |h_j W2_ij|
    w2d = deq(q["w2q"], q["s2"], orc)
    row_expert = ref["expert_of"][ref["assign_of_row"]]
    mag = np.stack([np.abs(w2d[e]) @ np.abs(deq(q["hq"][i], q["hs"][i], orc)) for i, e in
                    enumerate(row_expert)])
    step = np.stack([np.abs(w2d[e]) @ dh[i] for i, e in enumerate(row_expert)])
    ybound = step + 2.0 ** -16 * mag + 1e-30
    assert_within_bound(got["y"][:R], ref["y_rows"], ybound, "y")
    obound = np.zeros((w.N, w.d))
    for a in np.nonzero(ref["row_of"] >= 0)[0]:
        wa = abs(float(ref["topk_w"].reshape(-1)[a]))
        r = ref["row_of"][a]
        obound[a // w.K] += wa * ybound[r] + (w.K + 8) * 2.0 ** -24 * wa * np.abs(ref["y_rows"][r])
    assert_within_bound(got["out"], ref["out"], obound, "out")
    rep = tolerance_report(got["out"], ref["out"])
    assert rep["rel_frob"] <= 5e-3, rep
    if not moved.any():
        assert_within_tolerance(got["out"], ref["out"], "out")
    np.testing.assert_array_equal(got["out_layer"].cpu().numpy().view(np.uint32),
                                  got["out"].cpu().numpy().view(np.uint32))
    # the quantisation noise against the bf16 layer
    r16 = orc.layer(inp, w.K, w.W, w.cf, order=int(w.slot_major))
    dev = tolerance_report(got["out"], r16["out"])
    assert dev["rel_frob"] <= FP8_VS_BF16_REL_FROB, dev
    print(w.name, "fp8 vs bf16 layer", dev)


def test_fp8_down_gemm_on_oracle_rows(orc):
    """The e4m3 down GEMM fed the oracle's own e4m3 rows of h (and the oracle's quantised W2,
    which the GPU's quantiser reproduces bit for bit): every operand identical, so y may differ
    only by fp32 accumulation, checked element by element. Both kernels (pair tiles for the
    large experts, single-CTA for the small) and a 128-wide output tile (d = 384)."""
    m = lib()
    for w in (Workload("down_pair_split", N=3200, d=256, f=256, E=4, K=1, W=4, s=1.6),
              Workload("down_d384", N=384, d=384, f=256, E=6, K=3, W=3, cf=1.25, s=1.1)):
        inp = make_layer_inputs(w, seed=2)
        ref = orc.layer_fp8(inp, w.K, w.W, w.cf)
        q = ref["fp8"]
        shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf)
        RA = m.moe_rows_alloc(shape)
        R = ref["R"]
        hq = torch.zeros(RA, w.f, dtype=torch.uint8)
        hq[:R] = torch.from_numpy(q["hq"])
        hs = torch.zeros(RA, dtype=torch.float32)
        hs[:R] = torch.from_numpy(q["hs"])
        w2q, s2 = quantize_weights(m, inp["w2"].cuda())
        np.testing.assert_array_equal(_u8(w2q), q["w2q"])
        y = torch.zeros(RA, w.d, dtype=torch.float32, device="cuda")
        offsets = torch.from_numpy(ref["offsets"].astype(np.int32)).cuda()
        m.moe_expert_down_fp8(shape, hq.cuda(), hs.cuda(), offsets, w2q, s2, y)
        torch.cuda.synchronize()
        assert m.moe_get_device_error(True) == 0
        w2d = deq(q["w2q"], q["s2"], orc)
        row_expert = ref["expert_of"][ref["assign_of_row"]]
        mag = np.stack([np.abs(w2d[e]) @ np.abs(deq(q["hq"][i], q["hs"][i], orc)) for i, e in
                        enumerate(row_expert)])
        assert_within_bound(y[:R], ref["y_rows"], 2.0 ** -16 * mag + 1e-30, w.name)


def sampled_fp8_layer(orc, hx, K, toks, r, used, fp8_return=False):
    """The oracle's FP8 layer on sampled tokens: the quantised operands of the used experts,
    h and the e4m3 down projection for their kept rows (then, with fp8_return, the block
    quantisation of those rows of y), and the combine."""
    q = orc.fp8_operands(hx)
    remap = np.full(max(int(r["expert_of"].max()) + 1, 1), -1, np.int64)
    remap[used] = np.arange(len(used))
    slots = (toks[:, None] * K + np.arange(K)[None, :]).reshape(-1)
    kept = slots[r["row_of"][slots] >= 0]
    row_token = (kept // K).astype(np.int32)
    row_expert = remap[r["expert_of"][kept]].astype(np.int32)
    h, _ = orc.expert_rows(row_token, row_expert, q["x_deq"], q["w1_deq"], q["w3_deq"], hx["w2"],
                           True)
    y = orc.fp8_down(h, row_expert, q)["y"]
    if fp8_return:
        y = orc.dequantize_blocks_e4m3(*orc.quantize_blocks_e4m3(y))
    out = np.zeros((len(toks), y.shape[1]))
    pos = {int(a): i for i, a in enumerate(kept)}
    for li, t in enumerate(toks):
        for k in range(K):
            a = int(t) * K + k
            if a in pos:
                out[li] += float(r["topk_w"].reshape(-1)[a]) * y[pos[a]]
    return out, q


@pytest.mark.parametrize("fp8_return", [False, True], ids=["fp32_return", "fp8_return"])
def test_fp8_layer_full_size_mixtral(orc, fp8_return):
    """The Mixtral-shaped layer (N=4096, d=4096, f=14336, E=8, K=2) through moe_layer_fp8:
    routing in full, the weight codes of the used experts bit for bit, the output on sampled
    tokens against the oracle's FP8 layer (relative Frobenius bar) and against the bf16 layer
    (the FP8 bar); with and without the FP8 return payload."""
    from test_gpu_fullsize import host_inputs, sample_tokens
    m = lib()
    w = WORKLOADS["mixtral_prefill"]
    torch.cuda.empty_cache()
    inp = make_layer_inputs(w, seed=0, device="cuda")
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf, fp8_return=fp8_return)
    w1q, s1 = quantize_weights(m, inp["w1"])
    w3q, s3 = quantize_weights(m, inp["w3"])
    w2q, s2 = quantize_weights(m, inp["w2"])
    ws = torch.empty(m.moe_layer_workspace_size(shape), dtype=torch.uint8, device="cuda")
    out = torch.empty(w.N, w.d, dtype=torch.float32, device="cuda")
    topk = torch.empty(w.N, w.K, dtype=torch.int32, device="cuda")
    m.moe_layer_fp8(shape, inp["x"], inp["w_router"], inp["bias"], w1q, s1, w3q, s3, w2q, s2,
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
    ut = torch.from_numpy(used).cuda()
    hx = host_inputs(inp, experts=ut)
    got = out[torch.from_numpy(toks).cuda()]
    ref8, q = sampled_fp8_layer(orc, hx, w.K, toks, r, used, fp8_return)
    for name, qg, sg in (("w1q", w1q, s1), ("w3q", w3q, s3), ("w2q", w2q, s2)):
        np.testing.assert_array_equal(_u8(qg[ut]), q[name])
        np.testing.assert_array_equal(sg[ut].cpu().numpy(), q["s" + name[1]])
    rep = tolerance_report(got, ref8)
    assert rep["rel_frob"] <= 5e-3, rep
    rr = dict(r)
    remap = np.full(w.E, -1, np.int64)
    remap[used] = np.arange(len(used))
    rr["expert_of"] = np.where(r["expert_of"] >= 0, remap[r["expert_of"]], -1).astype(np.int32)
    smp16 = orc.layer_sampled(hx, w.K, w.W, w.cf, toks, routing=rr)
    dev = tolerance_report(got, smp16["out_tokens"])
    assert dev["rel_frob"] <= FP8_VS_BF16_REL_FROB, dev
    print("mixtral fp8", "fp8 return" if fp8_return else "", rep, "vs bf16", dev)
