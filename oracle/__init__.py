"""CPU oracle of the single-GPU MoE FFN layer (route -> dispatch -> SwiGLU
experts -> combine).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` (``cpu_baseline`` and ``--impl reference``) may import
this package. The product library never calls it, and it never calls the
product library: the two share no code.

The arithmetic lives in ``moe_oracle.c`` (plain loops, one function per step
of the method, each citing the page and section it restates). This module
compiles it with gcc, loads it with ctypes and marshals numpy arrays; the only
Python-side arithmetic is the host-side report (``derive_report``), written
out from its definitions below.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so beside it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-fvisibility=hidden", "-o", _LIB_PATH, _SRC, "-lm"]
    subprocess.check_call(cmd)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.orc_router_logits.argtypes = [_i64, _i64, _i64, _p, _p, _p, _p]
        lib.orc_router_logits.restype = None
        lib.orc_topk.argtypes = [_i64, _i64, _i64, _p, _p, _p]
        lib.orc_topk.restype = _i64
        lib.orc_capacity.argtypes = [_i64, _i64, _i64, ctypes.c_float]
        lib.orc_capacity.restype = _i64
        lib.orc_positions.argtypes = [_i64] * 5 + [_p] * 10
        lib.orc_positions.restype = None
        lib.orc_positions_ordered.argtypes = [_i64] * 6 + [_p] * 10
        lib.orc_positions_ordered.restype = None
        lib.orc_dispatch.argtypes = [_i64] * 7 + [_p] * 12
        lib.orc_dispatch.restype = None
        lib.orc_expert_rows.argtypes = [_i64, _p, _p, _i64, _i64, _p, _p, _p, _p, _p, _p]
        lib.orc_expert_rows.restype = None
        lib.orc_combine.argtypes = [_i64, _i64, _i64, _p, _p, _p, _p]
        lib.orc_combine.restype = None
        lib.orc_affinity.argtypes = [_i64, _i64, _i64, _p, _p, _p]
        lib.orc_affinity.restype = None
        lib.orc_e4m3_encode.argtypes = [_i64, _p, _p]
        lib.orc_e4m3_encode.restype = None
        lib.orc_e4m3_decode.argtypes = [_i64, _p, _p]
        lib.orc_e4m3_decode.restype = None
        lib.orc_e4m3_scale_exponent.argtypes = [ctypes.c_double]
        lib.orc_e4m3_scale_exponent.restype = _i64
        lib.orc_quantize_rows_e4m3.argtypes = [_i64, _i64, _p, _p, _p]
        lib.orc_quantize_rows_e4m3.restype = None
        lib.orc_quantize_blocks_e4m3.argtypes = [_i64, _i64, _i64, _p, _p, _p]
        lib.orc_quantize_blocks_e4m3.restype = None
        lib.orc_round_bf16.argtypes = [_i64, _p, _p]
        lib.orc_round_bf16.restype = None
        lib.orc_round_f16.argtypes = [_i64, _p, _p]
        lib.orc_round_f16.restype = None
        lib.orc_f16_scale_exponent.argtypes = [ctypes.c_double]
        lib.orc_f16_scale_exponent.restype = _i64
        lib.orc_quantize_blocks_f16.argtypes = [_i64, _i64, _i64, _p, _p, _p]
        lib.orc_quantize_blocks_f16.restype = None
        lib.orc_down_rows.argtypes = [_i64, _p, _i64, _i64, _p, _p, _p]
        lib.orc_down_rows.restype = None
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def as_u16(t) -> np.ndarray:
    """A bf16 torch tensor (or a uint16 array of bf16 bits) as contiguous uint16."""
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.uint16)
    import torch
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def as_f32(t) -> Optional[np.ndarray]:
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.float32)
    return t.detach().to("cpu").contiguous().float().numpy()


def bf16_bits_to_f64(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- steps

def router_logits(x, w_router, bias=None) -> np.ndarray:
    xs = as_u16(x)
    wr = as_f32(w_router)
    b = as_f32(bias)
    N, d = xs.shape
    E = wr.shape[0]
    out = np.empty((N, E), dtype=np.float32)
    _load().orc_router_logits(N, d, E, _ptr(xs), _ptr(wr), _ptr(b), _ptr(out))
    return out


def topk(logits: np.ndarray, K: int):
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    N, E = logits.shape
    idx = np.empty((N, K), dtype=np.int32)
    w = np.empty((N, K), dtype=np.float32)
    bad = _load().orc_topk(N, E, K, _ptr(logits), _ptr(idx), _ptr(w))
    return idx, w, int(bad)


def capacity(N: int, E: int, K: int, cf: float) -> int:
    return int(_load().orc_capacity(N, E, K, float(cf)))


SLOT_MAJOR = 1  # priority order of positions() / route_and_dispatch(): 0 token-major


def positions(topk_idx: np.ndarray, E: int, W: int, C: int, order: int = 0,
              reroute: bool = False, logits: Optional[np.ndarray] = None) -> dict:
    """Dispatch bookkeeping in priority ``order`` (0 token-major, SLOT_MAJOR), with
    overflowed assignments re-routed to the next-best non-full expert when
    ``reroute`` (then ``logits`` [N][E] fp32 rank the candidates)."""
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    N, K = topk_idx.shape
    if reroute:
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        assert logits.shape == (N, E)
    counts = np.empty(E, np.int32)
    kept = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    row_of = np.empty(N * K, np.int32)
    assign_of_row = np.full(N * K, -1, np.int32)
    expert_of = np.empty(N * K, np.int32)
    D = np.empty(W * W, np.int64)
    pk_off = np.empty(W * W + 1, np.int64)
    packed_row_of = np.empty(N * K, np.int32)
    stats = np.empty(9, np.int64)
    _load().orc_dispatch(N, E, K, W, C, order, int(bool(reroute)),
                         _ptr(logits) if reroute else None, _ptr(topk_idx), _ptr(counts),
                         _ptr(kept), _ptr(offsets), _ptr(row_of), _ptr(assign_of_row),
                         _ptr(expert_of), _ptr(D), _ptr(pk_off), _ptr(packed_row_of),
                         _ptr(stats))
    R = int(offsets[E])
    return dict(counts=counts, kept=kept, offsets=offsets, row_of=row_of,
                assign_of_row=assign_of_row[:R].copy(), expert_of=expert_of, D=D.reshape(W, W),
                pk_off=pk_off, packed_row_of=packed_row_of, R=R,
                stats=dict(R=int(stats[0]), dropped=int(stats[1]), cross_rows=int(stats[2]),
                           dedup_pairs=int(stats[3]), active_experts=int(stats[4]),
                           max_kept=int(stats[5]), min_kept=int(stats[6]), C=int(stats[7]),
                           rerouted=int(stats[8])))


def expert_rows(row_token: np.ndarray, row_expert: np.ndarray, x, w1, w3, w2,
                want_h: bool = False):
    row_token = np.ascontiguousarray(row_token, dtype=np.int32)
    row_expert = np.ascontiguousarray(row_expert, dtype=np.int32)
    xs, a, b, c = as_u16(x), as_u16(w1), as_u16(w3), as_u16(w2)
    d = xs.shape[1]
    f = a.shape[1]
    n = row_token.shape[0]
    y = np.empty((n, d), np.float64)
    h = np.empty((n, f), np.float64) if want_h else None
    _load().orc_expert_rows(n, _ptr(row_token), _ptr(row_expert), d, f, _ptr(xs), _ptr(a),
                            _ptr(b), _ptr(c), _ptr(h), _ptr(y))
    return h, y


def combine(row_of: np.ndarray, topk_w: np.ndarray, y_of_slot: np.ndarray) -> np.ndarray:
    """y_of_slot: [N*K][d] float64, the expert output of each (t, k) slot."""
    row_of = np.ascontiguousarray(row_of, dtype=np.int32).reshape(-1)
    topk_w = np.ascontiguousarray(topk_w, dtype=np.float32)
    N, K = topk_w.shape
    y_of_slot = np.ascontiguousarray(y_of_slot, dtype=np.float64)
    d = y_of_slot.shape[1]
    out = np.empty((N, d), np.float64)
    _load().orc_combine(N, K, d, _ptr(row_of), _ptr(topk_w), _ptr(y_of_slot), _ptr(out))
    return out


def affinity(topk_j: np.ndarray, topk_j1: np.ndarray, E: int,
             into: Optional[np.ndarray] = None) -> np.ndarray:
    a = np.ascontiguousarray(topk_j, dtype=np.int32)
    b = np.ascontiguousarray(topk_j1, dtype=np.int32)
    N, K = a.shape
    cnt = np.zeros((E, E), np.int64) if into is None else into
    _load().orc_affinity(N, E, K, _ptr(a), _ptr(b), _ptr(cnt))
    return cnt


# --------------------------------------------------------------------------- compositions

def route_and_dispatch(x, w_router, bias, K: int, W: int, cf: float, order: int = 0,
                       reroute: bool = False) -> dict:
    """Steps a1-a3: logits, top-K + weights, capacity, positions, layout."""
    logits = router_logits(x, w_router, bias)
    N, E = logits.shape
    idx, w, bad = topk(logits, K)
    C = capacity(N, E, K, cf)
    pos = positions(idx, E, W, C, order, reroute, logits)
    pos.update(logits=logits, topk_idx=idx, topk_w=w, nonfinite=bad, C=C)
    return pos


def layer(inp: dict, K: int, W: int, cf: float, want_h: bool = False, order: int = 0,
          reroute: bool = False) -> dict:
    """The whole layer on every token (small shapes only): returns the routing
    dict plus ``out`` [N][d] float64, ``y_rows`` [R][d] and optionally
    ``h_rows`` [R][f] (rows in expert-sorted order)."""
    r = route_and_dispatch(inp["x"], inp["w_router"], inp.get("bias"), K, W, cf, order, reroute)
    N = r["logits"].shape[0]
    aor = r["assign_of_row"]
    row_token = (aor // K).astype(np.int32)
    row_expert = r["expert_of"][aor].astype(np.int32)
    h, y = expert_rows(row_token, row_expert, inp["x"], inp["w1"], inp["w3"], inp["w2"], want_h)
    d = y.shape[1]
    y_of_slot = np.zeros((N * K, d), np.float64)
    kept = r["row_of"] >= 0
    y_of_slot[kept] = y[r["row_of"][kept]]
    r["out"] = combine(r["row_of"], r["topk_w"], y_of_slot)
    r["y_rows"] = y
    r["h_rows"] = h
    return r


def layer_sampled(inp: dict, K: int, W: int, cf: float, tokens: Sequence[int],
                  routing: Optional[dict] = None, want_h: bool = False) -> dict:
    """Routing and dispatch for every token; expert FFN and combine only for
    ``tokens``. Returns the routing dict plus ``out_tokens`` [n][d] (float64),
    and per kept slot of those tokens its expert-sorted row, y and h."""
    r = routing if routing is not None else route_and_dispatch(
        inp["x"], inp["w_router"], inp.get("bias"), K, W, cf)
    tokens = np.asarray(tokens, dtype=np.int64)
    slots = (tokens[:, None] * K + np.arange(K)[None, :]).reshape(-1)
    kept_slots = slots[r["row_of"][slots] >= 0]
    row_token = (kept_slots // K).astype(np.int32)
    row_expert = r["expert_of"][kept_slots].astype(np.int32)
    h, y = expert_rows(row_token, row_expert, inp["x"], inp["w1"], inp["w3"], inp["w2"], want_h)
    d = y.shape[1]
    n = tokens.shape[0]
    # combine restricted to the sampled tokens: re-index slots locally
    local_row_of = np.full(n * K, -1, np.int32)
    y_local = np.zeros((n * K, d), np.float64)
    pos_of_slot = {int(s): i for i, s in enumerate(kept_slots)}
    for li, t in enumerate(tokens):
        for k in range(K):
            s = int(t) * K + k
            if s in pos_of_slot:
                local_row_of[li * K + k] = 0
                y_local[li * K + k] = y[pos_of_slot[s]]
    w_local = r["topk_w"][tokens]
    out = combine(local_row_of, w_local, y_local)
    res = dict(r)
    res.update(out_tokens=out, sample_slots=kept_slots, sample_rows=r["row_of"][kept_slots],
               sample_y=y, sample_h=h)
    return res


def shared_expert(x, ws1, ws3, ws2) -> np.ndarray:
    """The shared dense MLP of a Residual-MoE layer on every token: the same SwiGLU form as an
    expert (W1s, W3s [f_s][d]; W2s [d][f_s]), computed by the expert routine with one expert
    that owns every row [MoE Inference Communication, §PR-MoE, 现象二 (Residual-MoE)]."""
    xs = as_u16(x)
    N = xs.shape[0]
    rows = np.arange(N, dtype=np.int32)
    _, y = expert_rows(rows, np.zeros(N, np.int32), xs, as_u16(ws1)[None], as_u16(ws3)[None],
                       as_u16(ws2)[None])
    return y


def layer_shared(inp: dict, shared: dict, K: int, W: int, cf: float, want_h: bool = False) -> dict:
    """Residual-MoE layer: out = (sum over kept slots of w_k * expert output) + shared MLP(x).
    [MoE Inference Communication, §PR-MoE: a shared dense MLP every token passes through plus
    routed experts, the two outputs added]"""
    r = layer(inp, K, W, cf, want_h)
    r["shared_y"] = shared_expert(inp["x"], shared["ws1"], shared["ws3"], shared["ws2"])
    r["out_routed"] = r["out"]
    r["out"] = r["out_routed"] + r["shared_y"]
    return r


# --------------------------------------------------------------------------- FP8 payload

def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Nearest e4m3 code of each value (ties to even, saturating at +-448)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint8)
    _load().orc_e4m3_encode(v.size, _ptr(v), _ptr(out))
    return out


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, np.float64)
    _load().orc_e4m3_decode(codes.size, _ptr(codes), _ptr(out))
    return out


def e4m3_scale_exponent(amax: float) -> int:
    return int(_load().orc_e4m3_scale_exponent(float(amax)))


def quantize_rows_e4m3(a) -> tuple:
    """Row-wise e4m3 quantisation of a bf16 matrix (torch bf16 or uint16 bits, any
    leading shape; rows are the last axis): (codes uint8, scale float32 per row)."""
    u = as_u16(a)
    shape = u.shape
    cols = shape[-1]
    rows = u.size // cols
    codes = np.empty(shape, np.uint8)
    scale = np.empty(shape[:-1], np.float32)
    _load().orc_quantize_rows_e4m3(rows, cols, _ptr(u), _ptr(codes), _ptr(scale))
    return codes, scale


def dequantize_rows_bf16(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """code value * row scale, as bf16 bits. Exact: an e4m3 value has 4 significant
    bits, bf16 has 8, and the scale is a power of two (asserted)."""
    v = e4m3_decode(codes) * scale.astype(np.float64)[..., None]
    f = v.astype(np.float32)
    bits = f.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0) and np.array_equal(f.astype(np.float64), v), \
        "dequantised value not exact in bf16"
    return (bits >> 16).astype(np.uint16)


def quantize_blocks_e4m3(v, block: int = 32) -> tuple:
    """Block-wise e4m3 quantisation of a float matrix [rows][cols] (fp32 or fp64 values, taken
    exactly): the row rule on every `block` consecutive columns. Returns (codes uint8
    [rows][cols], exps int32 [rows][cols / block]); value = code value * 2^exp."""
    a = np.ascontiguousarray(v, dtype=np.float64)
    rows, cols = a.shape
    assert cols % block == 0
    codes = np.empty((rows, cols), np.uint8)
    exps = np.empty((rows, cols // block), np.int32)
    _load().orc_quantize_blocks_e4m3(rows, cols, block, _ptr(a), _ptr(codes), _ptr(exps))
    return codes, exps


def round_f16(v: np.ndarray) -> np.ndarray:
    """Nearest fp16 of each float64 value (ties to even), as uint16 bits."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    _load().orc_round_f16(v.size, _ptr(v), _ptr(out))
    return out


def f16_scale_exponent(amax: float) -> int:
    return int(_load().orc_f16_scale_exponent(float(amax)))


def quantize_blocks_f16(v, block: int = 32) -> tuple:
    """Block-wise fp16 quantisation of a float matrix [rows][cols] (values taken exactly).
    Returns (codes uint16 fp16 bits [rows][cols], exps int32 [rows][cols / block]); value =
    fp16 code value * 2^exp."""
    a = np.ascontiguousarray(v, dtype=np.float64)
    rows, cols = a.shape
    assert cols % block == 0
    codes = np.empty((rows, cols), np.uint16)
    exps = np.empty((rows, cols // block), np.int32)
    _load().orc_quantize_blocks_f16(rows, cols, block, _ptr(a), _ptr(codes), _ptr(exps))
    return codes, exps


def dequantize_blocks_f16(codes: np.ndarray, exps: np.ndarray, block: int = 32) -> np.ndarray:
    """fp16 code value * 2^exp of every element, float64 (exact)."""
    v = np.asarray(codes, np.uint16).view(np.float16).astype(np.float64)
    return v * np.exp2(np.repeat(np.asarray(exps, np.float64), block, axis=1))


def dequantize_blocks_e4m3(codes: np.ndarray, exps: np.ndarray, block: int = 32) -> np.ndarray:
    """code value * 2^exp of every element, float64 (exact)."""
    v = e4m3_decode(codes)
    scale = np.ldexp(1.0, np.repeat(np.asarray(exps, dtype=np.int64), block, axis=-1))
    return v * scale


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Nearest bf16 of each float64 value (ties to even), as uint16 bits."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    _load().orc_round_bf16(v.size, _ptr(v), _ptr(out))
    return out


def down_rows(row_expert: np.ndarray, h_u16: np.ndarray, w2) -> np.ndarray:
    """y = W2[e] h for bf16 rows h [n][f] (uint16 bits), fp64."""
    row_expert = np.ascontiguousarray(row_expert, dtype=np.int32)
    h = np.ascontiguousarray(h_u16, dtype=np.uint16)
    c = as_u16(w2)
    n, f = h.shape
    d = c.shape[1]
    y = np.empty((n, d), np.float64)
    _load().orc_down_rows(n, _ptr(row_expert), d, f, _ptr(h), _ptr(c), _ptr(y))
    return y


def fp8_operands(inp: dict) -> dict:
    """The e4m3 operands of the FP8 expert GEMMs: x rows per token, W1, W3 and W2 rows per
    output channel, each with its power-of-two scale, and their exact bf16 dequantisations."""
    xq, sx = quantize_rows_e4m3(inp["x"])
    w1q, s1 = quantize_rows_e4m3(inp["w1"])
    w3q, s3 = quantize_rows_e4m3(inp["w3"])
    w2q, s2 = quantize_rows_e4m3(inp["w2"])
    return dict(xq=xq, sx=sx, w1q=w1q, s1=s1, w3q=w3q, s3=s3, w2q=w2q, s2=s2,
                x_deq=dequantize_rows_bf16(xq, sx), w1_deq=dequantize_rows_bf16(w1q, s1),
                w3_deq=dequantize_rows_bf16(w3q, s3), w2_deq=dequantize_rows_bf16(w2q, s2))


def fp8_down(h: np.ndarray, row_expert: np.ndarray, q: dict) -> dict:
    """The FP8 down projection: h rounded to bf16 (the precision it is stored in), its rows
    quantised to e4m3 with a power-of-two scale each, times the e4m3 W2 rows."""
    hb = round_bf16(h)
    hq, hs = quantize_rows_e4m3(hb)
    y = down_rows(row_expert, dequantize_rows_bf16(hq, hs), q["w2_deq"])
    return dict(h_bf16=hb, hq=hq, hs=hs, y=y)


def layer_fp8(inp: dict, K: int, W: int, cf: float, want_h: bool = False, order: int = 0,
              reroute: bool = False, fp8_return: bool = False) -> dict:
    """The layer with the FP8 payload and FP8 expert GEMMs: routing on the bf16 x; the
    gate/up projections on e4m3 rows of x (one scale per token) and e4m3 rows of W1, W3
    (one scale per output channel); h rounded to bf16, then its rows quantised to e4m3
    for the down projection with e4m3 rows of W2; the combine as in ``layer``. With
    ``fp8_return`` the expert outputs y travel back as e4m3 codes with one power-of-two
    exponent per 32-column block (``quantize_blocks_e4m3``) and the combine weighs their
    exact values."""
    q = fp8_operands(inp)
    r = route_and_dispatch(inp["x"], inp["w_router"], inp.get("bias"), K, W, cf, order, reroute)
    N = r["logits"].shape[0]
    aor = r["assign_of_row"]
    row_token = (aor // K).astype(np.int32)
    row_expert = r["expert_of"][aor].astype(np.int32)
    h, _ = expert_rows(row_token, row_expert, q["x_deq"], q["w1_deq"], q["w3_deq"], inp["w2"],
                       True)
    dn = fp8_down(h, row_expert, q)
    y = dn["y"]
    d = y.shape[1]
    if fp8_return:
        yq, ye = quantize_blocks_e4m3(y)
        r["y_payload"] = (yq, ye)
        r["y_exact"] = y
        y = dequantize_blocks_e4m3(yq, ye)
    y_of_slot = np.zeros((N * K, d), np.float64)
    kept = r["row_of"] >= 0
    y_of_slot[kept] = y[r["row_of"][kept]]
    r["out"] = combine(r["row_of"], r["topk_w"], y_of_slot)
    r["y_rows"] = y
    r["h_rows"] = h
    q.update(hq=dn["hq"], hs=dn["hs"], h_bf16=dn["h_bf16"])
    r["fp8"] = q
    return r


# --------------------------------------------------------------------------- report

def dispatch_bytes(rows: int, d: int, elem_bytes: int) -> int:
    """Payload of one dispatch: every routed row carries d elements
    [MoE Inference Communication, §横向对比 › 二、通信量级的差异]."""
    return int(rows) * int(d) * int(elem_bytes)


def derive_report(N: int, E: int, K: int, W: int, kept: np.ndarray, D: np.ndarray,
                  stats: dict, d: int, elem_bytes: int = 2) -> dict:
    """Observability figures, from their definitions:

    * drop rate = dropped / (N*K)                     [serving page §5.1]
    * per-rank send = row sums of D, recv = column sums; max/min ratios
                                                     [A2A page §可观测指标]
    * cross-rank fraction = kept rows leaving their home rank / kept rows
    * expert load per rank std/mean (population std) over ranks of recv
    * capacity_factor_effective = max_e kept[e] / (N*K/E)
    * tau_min (tokens) = max(max row sum, max col sum) of D without its
      diagonal (local tokens cross no link)          [Inference-Comm §Aurora 定理 4.2]
    """
    D = np.asarray(D, dtype=np.int64).reshape(W, W)
    send = D.sum(axis=1)
    recv = D.sum(axis=0)
    off = D.copy()
    np.fill_diagonal(off, 0)
    R = int(stats["R"])
    mean_recv = recv.mean()
    std_recv = math.sqrt(float(((recv - mean_recv) ** 2).mean()))
    tau = int(max(off.sum(axis=1).max(), off.sum(axis=0).max()))
    return dict(
        rows=R,
        dropped=int(stats["dropped"]),
        drop_rate=float(stats["dropped"]) / float(N * K),
        send_max=int(send.max()), send_min=int(send.min()),
        recv_max=int(recv.max()), recv_min=int(recv.min()),
        send_max_over_min=(float(send.max()) / float(send.min())) if send.min() > 0 else math.inf,
        recv_max_over_min=(float(recv.max()) / float(recv.min())) if recv.min() > 0 else math.inf,
        cross_rank_fraction=(float(stats["cross_rows"]) / R) if R > 0 else 0.0,
        dedup_pairs=int(stats["dedup_pairs"]),
        load_std_over_mean=(std_recv / mean_recv) if mean_recv > 0 else 0.0,
        capacity_factor_effective=float(np.max(kept)) / (float(N * K) / float(E)),
        tau_min_tokens=tau,
        dispatch_bytes=dispatch_bytes(R, d, elem_bytes),
        active_experts=int(stats["active_experts"]),
    )
