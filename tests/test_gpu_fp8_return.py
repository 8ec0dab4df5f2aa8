"""Parity of the FP8 return payload (expert outputs y as e4m3 codes with one power-of-two
exponent per 32-column block) with the oracle.

The quantisation decision is checked in the precision the kernel takes it in: the payload the
down GEMM writes must be, bit for bit, the oracle's block quantisation of the fp32 y the same
GEMM writes without the flag (the accumulation is deterministic, so the two launches quantise the
same values). The combine must weigh the payload's exact values (fp32 accumulation error only),
the fused layer must equal its stages bit for bit, and against the oracle's own FP8-return layer
(y in fp64, then quantised) codes differ only where the two y straddle an e4m3 rounding boundary.
"""
import numpy as np
import pytest
import torch

from layer_runner import assert_within_bound, lib, tolerance_report
from moe_workloads import WORKLOADS, Workload, make_layer_inputs
from test_gpu_fp8 import FP8_VS_BF16_REL_FROB, _u8, deq, quantize_weights, run_fp8_stages

pytestmark = pytest.mark.gpu


def split_payload(m, shape, buf, R):
    """(codes [R][d], exponents [R][d/32] as j, padding bytes [R][...]) of a payload buffer."""
    d = shape.d
    st = m.y_payload_stride(shape)
    rows = _u8(buf)[:m.moe_rows_alloc(shape) * st].reshape(-1, st)
    return (rows[:R, :d], rows[:R, d:d + d // 32].astype(np.int32) - 127, rows[:R, d + d // 32:],
            rows[R:])


# (name, E, rows per expert, d, f): pair tiles (>= 768 rows on average, d % 256 == 0),
# single-CTA 256-wide tiles with ragged experts, 128-wide tiles (d = 384), an empty expert
DOWN_CASES = [
    ("pair", 2, [1600, 900], 512, 256),
    ("ragged", 5, [1, 37, 0, 300, 129], 256, 384),
    ("d384", 3, [200, 5, 64], 384, 256),
]


@pytest.mark.parametrize("fp8_gemm", [False, True], ids=["bf16_down", "fp8_down"])
@pytest.mark.parametrize("case", DOWN_CASES, ids=[c[0] for c in DOWN_CASES])
def test_payload_is_the_block_code_of_y(orc, case, fp8_gemm):
    m = lib()
    name, E, rows, d, f = case
    R = sum(rows)
    N = -(-max(R, E) // E) * E
    # h and W2 in bf16 (the payload is quantised from whatever fp32 y the down GEMM forms)
    shape32 = m.make_shape(N, d, f, E, 1, 1, 0.0, h_bf16=True)
    shape8 = m.make_shape(N, d, f, E, 1, 1, 0.0, fp8_return=True, h_bf16=True)
    RA = m.moe_rows_alloc(shape32)
    assert RA >= R + 128
    g = torch.Generator().manual_seed(sum(map(ord, name)))
    # rows of h with magnitudes spread over many binades, a zero row
    h = (torch.randn(RA, f, generator=g) *
         torch.exp(torch.randn(RA, 1, generator=g) * 3)).to(torch.bfloat16)
    h[min(3, R - 1)] = 0.0
    w2 = (torch.randn(E, d, f, generator=g) * 0.02).to(torch.bfloat16).cuda()
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)).cuda()
    hc = h.cuda()
    y32 = torch.zeros(RA, d, dtype=torch.float32, device="cuda")
    pay = torch.full((m.moe_y_bytes(shape8),), 0xAB, dtype=torch.uint8, device="cuda")
    assert pay.numel() == RA * m.y_payload_stride(shape8)
    if fp8_gemm:
        hq = torch.empty(RA, f, dtype=torch.uint8, device="cuda")
        hs = torch.empty(RA, dtype=torch.float32, device="cuda")
        m.moe_quantize_rows_e4m3(hc, hq, hs)
        w2q, s2 = quantize_weights(m, w2)
        m.moe_expert_down_fp8(shape32, hq, hs, offsets, w2q, s2, y32)
        m.moe_expert_down_fp8(shape8, hq, hs, offsets, w2q, s2, pay)
    else:
        m.moe_expert_down(shape32, hc, offsets, w2, y32)
        m.moe_expert_down(shape8, hc, offsets, w2, pay)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(True) == 0
    codes, exps, pad, tail = split_payload(m, shape8, pay, R)
    rc, re = orc.quantize_blocks_e4m3(y32[:R].cpu().numpy())
    np.testing.assert_array_equal(exps, re)
    np.testing.assert_array_equal(codes, rc)
    assert np.all(pad == 0xAB) and np.all(tail == 0xAB), "bytes outside the kept rows written"


@pytest.mark.parametrize("N,d", [(96, 256), (2048, 256), (9600, 512)])
def test_combine_weighs_the_payload_exactly(orc, N, d):
    """moe_combine on a payload: out = sum_k w_k * (code * 2^j), fp32 accumulation in k order,
    then the shared MLP's output and the residual when given; the oracle's combine of the
    decoded payload (fp64) bounds the difference per element. N = 96 takes the sliced-row
    path (few tokens per SM), N = 2048 the whole-row path, N = 9600 with d = 512 the bulk-fed
    kernel (64 or more tokens per SM)."""
    m = lib()
    K, E = 3, 4
    shape = m.make_shape(N, d, 128, E, K, 1, 0.0, fp8_return=True)
    RA = m.moe_rows_alloc(shape)
    rng = np.random.default_rng(9)
    y = rng.standard_normal((RA, d)) * np.exp(rng.uniform(-8, 8, (RA, d // 32))).repeat(32, 1)
    codes, exps = orc.quantize_blocks_e4m3(y)
    st = m.y_payload_stride(shape)
    buf = np.zeros((RA, st), np.uint8)
    buf[:, :d] = codes
    buf[:, d:d + d // 32] = exps + 127
    row_of = rng.permutation(RA - 128)[:N * K].astype(np.int32)
    row_of[rng.random(N * K) < 0.15] = -1                    # dropped slots
    topk_w = rng.dirichlet(np.ones(K), N).astype(np.float32)
    deq_all = orc.dequantize_blocks_e4m3(codes, exps)
    y_of_slot = np.where(row_of[:, None] >= 0, deq_all[np.maximum(row_of, 0)], 0.0)
    ref = orc.combine(row_of, topk_w, y_of_slot)
    mag = orc.combine(row_of, np.abs(topk_w), np.abs(y_of_slot))
    # the extras a Residual-MoE layer and a stack add after the routed sum
    shared_y = (rng.standard_normal((N, d)) * 3).astype(np.float32)
    residual = torch.from_numpy(rng.standard_normal((N, d))).to(torch.bfloat16)
    res64 = residual.double().numpy()
    for out_bf16 in (False, True):
        for extras in (False, True):
            sh = m.make_shape(N, d, 128, E, K, 1, 0.0, out_bf16=out_bf16, fp8_return=True)
            out = torch.empty(N, d, dtype=torch.bfloat16 if out_bf16 else torch.float32,
                              device="cuda")
            m.moe_combine(sh, torch.from_numpy(buf.reshape(-1)).cuda(),
                          torch.from_numpy(row_of).cuda(), torch.from_numpy(topk_w).cuda(), out,
                          residual=residual.cuda() if extras else None,
                          shared_y=torch.from_numpy(shared_y).cuda() if extras else None)
            torch.cuda.synchronize()
            want = ref + (shared_y.astype(np.float64) + res64 if extras else 0.0)
            size = mag + (np.abs(shared_y) + np.abs(res64) if extras else 0.0)
            bound = ((K + 4) * 2.0 ** -24 * size + (2.0 ** -8 * np.abs(want) if out_bf16 else 0)
                     + 1e-37)
            assert_within_bound(out.float(), want, bound, f"out_bf16={out_bf16} extras={extras}")


CASES = [
    Workload("fp8r_small", N=64, d=128, f=256, E=8, K=2, W=4),
    Workload("fp8r_drop", N=384, d=384, f=256, E=6, K=3, W=3, cf=1.25, s=1.1),
    Workload("fp8r_pair", N=1600, d=512, f=256, E=2, K=1, W=2),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_fp8_return_layer(orc, w):
    """The whole FP8 layer with the FP8 return payload: the fused entry point equals the
    stages bit for bit; the output equals the combine of the GPU's own payload; the payload's
    codes equal the oracle's (y in fp64, then quantised) except where the two y straddle a
    rounding boundary (rare), within the bound the arithmetic gives; the output meets the
    relative-Frobenius bar against the oracle's FP8-return layer and the FP8 bar against the
    bf16 layer."""
    m = lib()
    inp = make_layer_inputs(w, seed=3)
    ref = orc.layer_fp8(inp, w.K, w.W, w.cf, fp8_return=True)
    got = run_fp8_stages(inp, w, fp8_return=True)
    assert got["dev_error"] == 0
    np.testing.assert_array_equal(got["out_layer"].cpu().numpy().view(np.uint32),
                                  got["out"].cpu().numpy().view(np.uint32))
    R = ref["R"]
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf, fp8_return=True)
    codes, exps, _, _ = split_payload(m, shape, got["y"], R)
    # the output is the combine of the payload the GPU wrote
    deq_g = orc.dequantize_blocks_e4m3(codes, exps)
    kept = ref["row_of"] >= 0
    y_of_slot = np.zeros((w.N * w.K, w.d))
    y_of_slot[kept] = deq_g[ref["row_of"][kept]]
    own = orc.combine(ref["row_of"], got["topk_w"].cpu().numpy(), y_of_slot)
    mag = orc.combine(ref["row_of"], np.abs(got["topk_w"].cpu().numpy()), np.abs(y_of_slot))
    assert_within_bound(got["out"], own, (w.K + 2) * 2.0 ** -24 * mag + 1e-37, "combine")
    # against the oracle's payload (its y in fp64, then quantised): codes agree except where
    # the two y straddle a rounding boundary (rare), and every decoded value lies within the
    # two quantisation half-steps of the difference between the two y that the arithmetic
    # bounds (h's e4m3 codes that moved, fp32 accumulation), as for fp32 y
    oq, oe = ref["y_payload"]
    moved = codes != oq
    assert moved.mean() <= 1e-3, moved.mean()
    q = ref["fp8"]
    hq_gpu, hs_gpu = _u8(got["hq"])[:R], got["hs"].cpu().numpy()[:R]
    dh = np.abs(deq(hq_gpu, hs_gpu, orc) - deq(q["hq"], q["hs"], orc))
    w2d = deq(q["w2q"], q["s2"], orc)
    row_expert = ref["expert_of"][ref["assign_of_row"]]
    mag = np.stack([np.abs(w2d[e]) @ np.abs(deq(q["hq"][i], q["hs"][i], orc)) for i, e in
                    enumerate(row_expert)])
    step = np.stack([np.abs(w2d[e]) @ dh[i] for i, e in enumerate(row_expert)])
    ybound = step + 2.0 ** -16 * mag + 1e-30
    deq_o = orc.dequantize_blocks_e4m3(oq, oe)

    def half_step(v, e):  # |code value * 2^j - y| for the y it came from (normal / subnormal)
        return 0.07 * np.abs(v) + np.ldexp(1.0, np.repeat(e, 32, axis=1) - 10)

    assert_within_bound(deq_g, deq_o, ybound + half_step(deq_g, exps) + half_step(deq_o, oe),
                        "payload")
    rep = tolerance_report(got["out"], ref["out"])
    assert rep["rel_frob"] <= 5e-3, rep
    r16 = orc.layer(inp, w.K, w.W, w.cf)
    dev = tolerance_report(got["out"], r16["out"])
    assert dev["rel_frob"] <= FP8_VS_BF16_REL_FROB, dev
    print(w.name, "fp8 return vs oracle", rep, "vs bf16", dev)
