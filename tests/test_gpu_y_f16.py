"""Parity of the fp16 return payload (expert outputs y as fp16 codes with one power-of-two
exponent per 32-column block, MOE_FLAG_Y_F16) with the oracle.

The quantisation decision is checked in the precision the kernel takes it in: the payload the
down GEMM writes must be, bit for bit, the oracle's fp16 block quantisation of the fp32 y the same
GEMM writes without the flag (the accumulation is deterministic). The combine must weigh the
payload's exact values (fp32 accumulation error only), the fused layer must equal its stages bit
for bit, and the layer output must meet the stated bar against the oracle's fp64 layer.
"""
import numpy as np
import pytest
import torch

from layer_runner import assert_within_bound, lib, run_layer, run_stages, tolerance_report
from moe_workloads import Workload, make_layer_inputs
from test_gpu_fp8 import _u8, quantize_weights

pytestmark = pytest.mark.gpu


def split_payload(m, shape, buf, R):
    """(codes as fp16 bits [R][d], exponents [R][d/32] as j, padding bytes, rows past R)."""
    d = shape.d
    st = m.y_payload_stride(shape)
    rows = _u8(buf)[:m.moe_rows_alloc(shape) * st].reshape(-1, st)
    codes = np.ascontiguousarray(rows[:R, :2 * d]).view(np.uint16)
    return (codes, rows[:R, 2 * d:2 * d + d // 32].astype(np.int32) - 127,
            rows[:R, 2 * d + d // 32:], rows[R:])


# (name, E, rows per expert, d, f): pair tiles (>= 768 rows on average, d % 256 == 0),
# single-CTA 256-wide tiles with ragged experts, 128-wide tiles (d = 384), an empty expert
DOWN_CASES = [
    ("pair", 2, [1600, 900], 512, 256),
    ("ragged", 5, [1, 37, 0, 300, 129], 256, 384),
    ("d384", 3, [200, 5, 64], 384, 256),
]


@pytest.mark.parametrize("gemm", ["f16_h", "bf16_h", "fp8"])
@pytest.mark.parametrize("case", DOWN_CASES, ids=[c[0] for c in DOWN_CASES])
def test_payload_is_the_block_code_of_y(orc, case, gemm):
    m = lib()
    name, E, rows, d, f = case
    R = sum(rows)
    N = -(-max(R, E) // E) * E
    h_bf16 = gemm == "bf16_h"
    shape32 = m.make_shape(N, d, f, E, 1, 1, 0.0, h_bf16=h_bf16)
    shape16 = m.make_shape(N, d, f, E, 1, 1, 0.0, h_bf16=h_bf16, y_f16=True)
    RA = m.moe_rows_alloc(shape32)
    assert RA >= R + 128
    g = torch.Generator().manual_seed(sum(map(ord, name)) + 16)
    # rows of h with magnitudes spread over many binades (within fp16's range), a zero row
    h = torch.randn(RA, f, generator=g) * torch.exp(torch.randn(RA, 1, generator=g) * 2)
    h[min(3, R - 1)] = 0.0
    h[RA - 1] = 0.0  # the fp16 range word of h's buffer: in range (no rescaling)
    hc = h.to(torch.bfloat16 if h_bf16 or gemm == "fp8" else torch.float16).cuda()
    w2b = (torch.randn(E, d, f, generator=g) * 0.02).to(torch.bfloat16).cuda()
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)).cuda()
    y32 = torch.zeros(RA, d, dtype=torch.float32, device="cuda")
    pay = torch.full((m.moe_y_bytes(shape16),), 0xAB, dtype=torch.uint8, device="cuda")
    assert pay.numel() == RA * m.y_payload_stride(shape16)
    if gemm == "fp8":
        hq = torch.empty(RA, f, dtype=torch.uint8, device="cuda")
        hs = torch.empty(RA, dtype=torch.float32, device="cuda")
        m.moe_quantize_rows_e4m3(hc, hq, hs)
        w2q, s2 = quantize_weights(m, w2b)
        m.moe_expert_down_fp8(shape32, hq, hs, offsets, w2q, s2, y32)
        m.moe_expert_down_fp8(shape16, hq, hs, offsets, w2q, s2, pay)
    else:
        w2 = m.w2_for(shape32, w2b)
        m.moe_expert_down(shape32, hc, offsets, w2, y32)
        m.moe_expert_down(shape16, hc, offsets, w2, pay)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(True) == 0
    codes, exps, pad, tail = split_payload(m, shape16, pay, R)
    rc, re = orc.quantize_blocks_f16(y32[:R].cpu().numpy())
    np.testing.assert_array_equal(exps, re)
    np.testing.assert_array_equal(codes, rc)
    assert np.all(pad == 0xAB) and np.all(tail == 0xAB), "bytes outside the kept rows written"


@pytest.mark.parametrize("N,d", [(96, 256), (2048, 256), (9600, 512)])
def test_combine_weighs_the_payload_exactly(orc, N, d):
    """moe_combine on an fp16 payload: out = sum_k w_k * (code * 2^j), fp32 accumulation in k
    order, then the shared MLP's output and the residual when given; the oracle's combine of
    the decoded payload (fp64) bounds the difference per element. N = 96 takes the sliced-row
    path, N = 2048 the whole-row path, N = 9600 with d = 512 the bulk-fed kernel
    (64 or more tokens per SM)."""
    m = lib()
    K, E = 3, 4
    shape = m.make_shape(N, d, 128, E, K, 1, 0.0, y_f16=True)
    RA = m.moe_rows_alloc(shape)
    rng = np.random.default_rng(19)
    y = rng.standard_normal((RA, d)) * np.exp(rng.uniform(-12, 12, (RA, d // 32))).repeat(32, 1)
    codes, exps = orc.quantize_blocks_f16(y)
    st = m.y_payload_stride(shape)
    buf = np.zeros((RA, st), np.uint8)
    buf[:, :2 * d] = codes.view(np.uint8).reshape(RA, 2 * d)
    buf[:, 2 * d:2 * d + d // 32] = exps + 127
    row_of = rng.permutation(RA - 128)[:N * K].astype(np.int32)
    row_of[rng.random(N * K) < 0.15] = -1                    # dropped slots
    topk_w = rng.dirichlet(np.ones(K), N).astype(np.float32)
    deq_all = orc.dequantize_blocks_f16(codes, exps)
    y_of_slot = np.where(row_of[:, None] >= 0, deq_all[np.maximum(row_of, 0)], 0.0)
    ref = orc.combine(row_of, topk_w, y_of_slot)
    mag = orc.combine(row_of, np.abs(topk_w), np.abs(y_of_slot))
    shared_y = (rng.standard_normal((N, d)) * 3).astype(np.float32)
    residual = torch.from_numpy(rng.standard_normal((N, d))).to(torch.bfloat16)
    res64 = residual.double().numpy()
    for out_bf16 in (False, True):
        for extras in (False, True):
            sh = m.make_shape(N, d, 128, E, K, 1, 0.0, out_bf16=out_bf16, y_f16=True)
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
    Workload("y16_small", N=64, d=128, f=256, E=8, K=2, W=4),
    Workload("y16_drop", N=384, d=384, f=256, E=6, K=3, W=3, cf=1.25, s=1.1),
    Workload("y16_sparse", N=256, d=128, f=128, E=64, K=6, W=8, cf=1.0, s=1.2),
    Workload("y16_pair", N=1600, d=512, f=256, E=2, K=1, W=2),
    Workload("y16_slot_reroute", N=1040, d=256, f=384, E=8, K=2, W=4, cf=0.8, s=0.8,
             slot_major=True, reroute=True),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_y_f16_layer(orc, w):
    """The layer with the fp16 payload: the fused entry point equals the stages bit for bit;
    the output equals the combine of the GPU's own payload (fp32 accumulation); the output meets
    the stated bar (relative Frobenius 5e-3, max-abs 2e-2 RMS) against the oracle's fp64 layer;
    and the payload's decoded values are the GPU's own fp32 y within half an fp16 step."""
    m = lib()
    inp = make_layer_inputs(w, seed=4)
    ref = orc.layer(inp, w.K, w.W, w.cf, order=int(w.slot_major), reroute=w.reroute)
    got = run_stages(inp, w, y_f16=True)
    assert got["dev_error"] == 0
    lay = run_layer(inp, w, y_f16=True)
    assert lay["dev_error"] == 0
    np.testing.assert_array_equal(lay["out"].cpu().numpy().view(np.uint32),
                                  got["out"].cpu().numpy().view(np.uint32))
    R = int(got["offsets"][w.E].item())
    assert R == ref["R"]
    shape = got["shape"]
    codes, exps, _, _ = split_payload(m, shape, got["y"], R)
    deq_g = orc.dequantize_blocks_f16(codes, exps)
    row_of = got["row_of"].cpu().numpy()
    kept = row_of >= 0
    y_of_slot = np.zeros((w.N * w.K, w.d))
    y_of_slot[kept] = deq_g[row_of[kept]]
    tw = got["topk_w"].cpu().numpy()
    own = orc.combine(row_of, tw, y_of_slot)
    mag = orc.combine(row_of, np.abs(tw), np.abs(y_of_slot))
    assert_within_bound(got["out"], own, (w.K + 2) * 2.0 ** -24 * mag + 1e-37, "combine")
    # the same layer with fp32 y: its y is what the payload encodes
    g32 = run_stages(inp, w)
    y32 = g32["y"][:R].cpu().numpy().astype(np.float64)
    scale = np.exp2(np.repeat(exps, 32, axis=1).astype(np.float64))
    assert np.all(np.abs(deq_g - y32) <= 2.0 ** -11 * np.maximum(np.abs(y32), 2.0 ** -14 * scale))
    rep = tolerance_report(got["out"], ref["out"])
    assert rep["rel_frob"] <= 5e-3 and rep["max_abs_over_rms"] <= 2e-2, rep
    print(w.name, "y fp16 payload vs oracle", rep)
