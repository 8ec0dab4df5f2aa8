"""Runs the CUDA path stage by stage (through the C ABI) and holds the results
as host arrays, plus the tolerance checks the parity tests share."""
from __future__ import annotations

import numpy as np
import torch


def lib():
    from combine_grouped_gemm_router_b200 import build
    build.build()
    import combine_grouped_gemm_router_b200 as m
    return m


def run_stages(inp: dict, w, pack: bool = True, device: str = "cuda", h_bf16: bool = False,
               y_f16: bool = False) -> dict:
    """route -> dispatch -> expert GEMMs -> combine, each through its C entry point. h and the
    down-projection weights are fp16 (the library's default) unless h_bf16; y is fp32, or the
    fp16 payload (uint8 bytes) with y_f16."""
    m = lib()
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf, slot_major=w.slot_major,
                         reroute=w.reroute, h_bf16=h_bf16, y_f16=y_f16)
    dev = torch.device(device)
    x = inp["x"].to(dev)
    wr = inp["w_router"].to(dev)
    bias = None if inp["bias"] is None else inp["bias"].to(dev)
    N, K, E, W, d, f = w.N, w.K, w.E, w.W, w.d, w.f
    RA = m.moe_rows_alloc(shape)
    ws = torch.empty(max(m.moe_workspace_size(shape), 256), dtype=torch.uint8, device=dev)
    logits = torch.empty(N, E, dtype=torch.float32, device=dev)
    topk_idx = torch.empty(N, K, dtype=torch.int32, device=dev)
    topk_w = torch.empty(N, K, dtype=torch.float32, device=dev)
    m.moe_route(shape, x, wr, bias, topk_idx, topk_w, logits, ws)

    counts = torch.empty(E, dtype=torch.int32, device=dev)
    kept = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty(N * K, dtype=torch.int32, device=dev)
    assign = torch.full((RA,), -7, dtype=torch.int32, device=dev)
    x_sorted = torch.zeros(RA, d, dtype=torch.bfloat16, device=dev)
    x_packed = torch.zeros(RA, d, dtype=torch.bfloat16, device=dev) if pack else None
    D = torch.empty(W * W, dtype=torch.int64, device=dev)
    pk_off = torch.empty(W * W + 1, dtype=torch.int64, device=dev)
    stats = m.stats_buffer(dev)
    expert_of = None
    if w.reroute:
        expert_of = torch.full((N * K,), -7, dtype=torch.int32, device=dev)
        m.moe_dispatch_reroute(shape, x, logits, topk_idx, counts, kept, offsets, row_of, assign,
                               x_sorted, expert_of=expert_of, x_packed=x_packed, rank_matrix=D,
                               packed_offsets=pk_off, stats=stats, ws=ws)
    else:
        m.moe_dispatch(shape, x, topk_idx, counts, kept, offsets, row_of, assign, x_sorted,
                       x_packed, D, pk_off, stats, ws)
    res = dict(shape=shape, logits=logits, topk_idx=topk_idx, topk_w=topk_w, counts=counts,
               kept=kept, offsets=offsets, row_of=row_of, assign=assign, x_sorted=x_sorted,
               x_packed=x_packed, D=D, pk_off=pk_off, stats_buf=stats, rows_alloc=RA,
               expert_of=expert_of)
    if w.d % 128 == 0 and w.f % 128 == 0:
        h = torch.zeros(RA, f, dtype=torch.bfloat16 if h_bf16 else torch.float16, device=dev)
        y = (torch.zeros(m.moe_y_bytes(shape), dtype=torch.uint8, device=dev) if y_f16 else
             torch.zeros(RA, d, dtype=torch.float32, device=dev))
        w2 = m.w2_for(shape, inp["w2"].to(dev))
        m.moe_expert_gemm(shape, x_sorted, offsets, inp["w1"].to(dev), inp["w3"].to(dev),
                          w2, h, y)
        out = torch.empty(N, d, dtype=torch.float32, device=dev)
        m.moe_combine(shape, y, row_of, topk_w, out)
        res.update(h=h, y=y, out=out, w2_used=w2)
    torch.cuda.synchronize()
    res["stats"] = m.stats_dict(m.read_stats(stats))
    res["dev_error"] = m.moe_get_device_error(True)
    return res


def run_layer(inp: dict, w, device: str = "cuda", with_stats: bool = True,
              h_bf16: bool = False, y_f16: bool = False) -> dict:
    m = lib()
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf, slot_major=w.slot_major,
                         reroute=w.reroute, h_bf16=h_bf16, y_f16=y_f16)
    dev = torch.device(device)
    ws = torch.empty(m.moe_layer_workspace_size(shape), dtype=torch.uint8, device=dev)
    out = torch.empty(w.N, w.d, dtype=torch.float32, device=dev)
    topk = torch.empty(w.N, w.K, dtype=torch.int32, device=dev)
    stats = m.stats_buffer(dev) if with_stats else None
    bias = None if inp["bias"] is None else inp["bias"].to(dev)
    m.moe_layer(shape, inp["x"].to(dev), inp["w_router"].to(dev), bias, inp["w1"].to(dev),
                inp["w3"].to(dev), m.w2_for(shape, inp["w2"].to(dev)), out, topk_idx_out=topk,
                stats=stats, ws=ws)
    torch.cuda.synchronize()
    res = dict(out=out, topk_idx=topk, ws=ws)
    if with_stats:
        res["stats"] = m.stats_dict(m.read_stats(stats))
    res["dev_error"] = m.moe_get_device_error(True)
    return res


def decode_y_payload(shape, ybuf, rows) -> np.ndarray:
    """Rows `rows` of an fp16 return payload (uint8 bytes on the device) decoded to fp64:
    code * 2^j per 32-column block."""
    m = lib()
    d, st = shape.d, m.y_payload_stride(shape)
    b = ybuf[:m.moe_rows_alloc(shape) * st].view(-1, st)[rows].cpu().numpy()
    codes = np.ascontiguousarray(b[:, :2 * d]).view(np.float16).astype(np.float64)
    j = b[:, 2 * d:2 * d + d // 32].astype(np.int64) - 127
    return codes * np.exp2(np.repeat(j, 32, axis=1).astype(np.float64))


def f16_payload_bound(ybound, y_ref) -> np.ndarray:
    """ybound (the fp32 y's distance from the oracle's y_ref) widened by the rounding of y to
    the fp16 block payload: half an fp16 step of |y|, or, where y is subnormal at the block's
    scale 2^j, half the smallest step there (j is the smallest with blockmax * 2^-j <= 65504,
    so 2^j < 2 * blockmax / 65504; j >= -126)."""
    top = np.abs(f64(y_ref)) + ybound
    bm = top.reshape(*top.shape[:-1], -1, 32).max(-1)
    s = np.maximum(2.0 * bm / 65504.0, 2.0 ** -126)
    return ybound + 2.0 ** -11 * top + 2.0 ** -25 * np.repeat(s, 32, axis=-1)


def f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().float().cpu().numpy().astype(np.float64)


def tolerance_report(got, ref) -> dict:
    """Relative Frobenius error and max-abs error / RMS(ref)."""
    g = f64(got)
    r = f64(ref)
    err = g - r
    nr = np.linalg.norm(r)
    rms = np.sqrt(np.mean(r * r)) if r.size else 0.0
    return dict(rel_frob=float(np.linalg.norm(err) / nr) if nr > 0 else float(np.linalg.norm(err)),
                max_abs_over_rms=float(np.max(np.abs(err)) / rms) if rms > 0 else 0.0)


# The stated bar for floating-point outputs against the oracle.
REL_FROB = 5e-3
MAX_ABS_OVER_RMS = 2e-2


def assert_rounded_bf16(got, ref, what: str = ""):
    """An intermediate stored as bf16: each element within one bf16 rounding
    (2^-8 relative) of the reference plus fp32 accumulation slack."""
    g = f64(got)
    r = f64(ref)
    rms = np.sqrt(np.mean(r * r))
    excess = np.abs(g - r) - (2.0 ** -8 * np.abs(r) + 1e-3 * rms)
    assert excess.max() <= 0, (what, float(excess.max() / rms))
    assert tolerance_report(g, r)["rel_frob"] <= REL_FROB, what


def assert_rounded_f16(got, ref, what: str = "", d: int = 128):
    """An intermediate stored as fp16: each element within twice fp16's rounding (2^-10
    relative; 11 significant bits) of the reference, plus half the subnormal step (2^-25) and
    a slack of d * 2^-24 * RMS for the two fp32 dot products over d terms that feed it (the
    gate and the up projection) and the SwiGLU's fp32 arithmetic. That slack is the usual
    worst-case growth of fp32 summation error over d terms, relative to the typical size of
    the result; it stays below fp16's own relative step for d < 8192."""
    g = f64(got)
    r = f64(ref)
    rms = np.sqrt(np.mean(r * r))
    excess = np.abs(g - r) - (2.0 ** -10 * np.abs(r) + 2.0 ** -25 + max(d, 128) * 2.0 ** -24 * rms)
    assert excess.max() <= 0, (what, float(excess.max() / rms))
    assert tolerance_report(g, r)["rel_frob"] <= REL_FROB, what


def assert_rounded_h(got, ref, what: str = "", d: int = 128):
    """h as the GPU stores it: fp16 by default, bf16 with the h_bf16 flag; d is the length of
    the dot products that produced it."""
    if got.dtype == torch.float16:
        assert_rounded_f16(got, ref, what, d)
    else:
        assert_rounded_bf16(got, ref, what)


def bf16_h_bound_rows(h_ref: np.ndarray, w2_f64: np.ndarray, row_expert: np.ndarray) -> np.ndarray:
    """Per-element bound on |y_gpu - y_ref| implied by the arithmetic: h is rounded once
    to bf16 (relative error <= 2^-8) before the down projection, which accumulates in
    fp32 over f terms: |dy_i| <= (2^-8 + f*2^-23) * sum_j |h_j W2[i][j]| (+ tiny)."""
    f = h_ref.shape[1]
    bound = np.empty((h_ref.shape[0], w2_f64.shape[1]))
    for e in np.unique(row_expert):
        sel = row_expert == e
        bound[sel] = np.abs(h_ref[sel]) @ np.abs(w2_f64[e]).T
    return bound * (2.0 ** -8 + f * 2.0 ** -23) + 1e-30


def f16_h_bound_rows(h_ref: np.ndarray, w2_f64: np.ndarray, w2_used_f64: np.ndarray,
                     row_expert: np.ndarray) -> np.ndarray:
    """The same bound for the default precision: h rounded once to fp16 (relative error
    <= 2^-11, bounded by 2^-10; absolute error <= 2^-25 where h is subnormal) and the fp16 copy
    of W2 (w2_used_f64, the weights the GPU multiplied; it differs from W2 only where a bf16
    weight is not an fp16 value): |dy_i| <= (2^-10 + f*2^-23) * sum_j |h_j W2[i][j]|
    + 2^-25 * sum_j |W2[i][j]| + sum_j |h_j| |W2_used[i][j] - W2[i][j]| (+ tiny)."""
    f = h_ref.shape[1]
    bound = np.empty((h_ref.shape[0], w2_f64.shape[1]))
    for e in np.unique(row_expert):
        sel = row_expert == e
        ah = np.abs(h_ref[sel])
        a2 = np.abs(w2_f64[e])
        bound[sel] = ((2.0 ** -10 + f * 2.0 ** -23) * (ah @ a2.T) + 2.0 ** -25 * a2.sum(1)[None]
                      + ah @ np.abs(w2_used_f64[e] - w2_f64[e]).T)
    return bound + 1e-30


def h_bound_rows(h_ref, inp_w2, got_w2_used, row_expert) -> np.ndarray:
    """The per-element y bound for the precision the run used (fp16 h unless the run kept W2
    in bf16)."""
    w2 = f64(inp_w2)
    if got_w2_used is None or got_w2_used.dtype == torch.bfloat16:
        return bf16_h_bound_rows(h_ref, w2, row_expert)
    return f16_h_bound_rows(h_ref, w2, f64(got_w2_used), row_expert)


def assert_within_bound(got, ref, bound, what: str = ""):
    g, r = f64(got), f64(ref)
    err = np.abs(g - r)
    ratio = err / np.maximum(bound, 1e-30)
    i = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
    worst = float(ratio[i])
    rms = float(np.sqrt(np.mean(r * r))) or 1.0
    assert worst <= 1.0, (what, dict(worst=worst, at=tuple(int(v) for v in i), got=float(g[i]),
                                     ref=float(r[i]), bound=float(bound[i]),
                                     err_over_rms=float(err[i] / rms)))
    return worst


def assert_within_tolerance(got, ref, what: str = ""):
    rep = tolerance_report(got, ref)
    assert rep["rel_frob"] <= REL_FROB and rep["max_abs_over_rms"] <= MAX_ABS_OVER_RMS, (what, rep)
    return rep
