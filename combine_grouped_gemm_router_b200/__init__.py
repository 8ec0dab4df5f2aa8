"""Python binding of the B200 MoE layer library (``libmoe_b200.so``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels, and the exchange planning (moe_exchange_schedule, moe_place_experts,
moe_place_experts_staged, moe_placement_order) in its host code. Torch tensors
supply device memory and the current stream; the planning functions take and
return numpy arrays. The functions keep the C names of ``include/moe_b200.h``;
each raises ``MoeError`` on a non-OK status. ``exchange`` (a submodule) moves
packed rows between ranks with torch.distributed. There is no fallback: the first call raises
``ImportError`` when the library has not been built
(``python -m combine_grouped_gemm_router_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_b200.so")


c_i32, c_i64, c_u32, c_u64, c_f32 = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                     ctypes.c_uint64, ctypes.c_float)
c_size, c_p = ctypes.c_size_t, ctypes.c_void_p

MOE_OK = 0
STATUS_NAMES = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_MISALIGNED", 5: "MOE_ERR_CUDA",
    6: "MOE_ERR_DEVICE_TIMEOUT", 7: "MOE_ERR_NONFINITE", 8: "MOE_ERR_DEVICE_BOUNDS",
    9: "MOE_ERR_F16_RANGE",
}


class MoeShape(ctypes.Structure):
    _fields_ = [("N", c_i32), ("d", c_i32), ("f", c_i32), ("E", c_i32), ("K", c_i32),
                ("W", c_i32), ("capacity_factor", c_f32), ("flags", c_u32)]


class MoeStats(ctypes.Structure):
    _fields_ = [("rows", c_i64), ("dropped", c_i64), ("cross_rows", c_i64),
                ("dedup_pairs", c_i64), ("nonfinite_tokens", c_i64), ("capacity", c_i32),
                ("active_experts", c_i32), ("max_kept", c_i32), ("min_kept", c_i32),
                ("rerouted", c_i64)]


class MoeReport(ctypes.Structure):
    _fields_ = [("drop_rate", ctypes.c_double), ("send_max_over_min", ctypes.c_double),
                ("recv_max_over_min", ctypes.c_double), ("cross_rank_fraction", ctypes.c_double),
                ("load_std_over_mean", ctypes.c_double),
                ("capacity_factor_effective", ctypes.c_double), ("tau_min_tokens", c_i64),
                ("dispatch_bytes", c_i64), ("send_max", c_i64), ("send_min", c_i64),
                ("recv_max", c_i64), ("recv_min", c_i64)]


_SP = ctypes.POINTER(MoeShape)
_sigs = {
    "moe_abi_version": ([], c_i32),
    "moe_status_string": ([c_i32], ctypes.c_char_p),
    "moe_capacity": ([_SP], c_i64),
    "moe_rows_alloc": ([_SP], c_i64),
    "moe_workspace_size": ([_SP], c_size),
    "moe_layer_workspace_size": ([_SP], c_size),
    "moe_y_bytes": ([_SP], c_size),
    "moe_route": ([_SP] + [c_p] * 7 + [c_size, c_p], c_i32),
    "moe_dispatch": ([_SP] + [c_p] * 13 + [c_size, c_p], c_i32),
    "moe_dispatch_static": ([_SP] + [c_p] * 13, c_i32),
    "moe_dispatch_rank": ([_SP, c_i32] + [c_p] * 14 + [c_size, c_p], c_i32),
    "moe_regroup_rows": ([_SP, c_i32, c_i32, c_i32] + [c_p] * 8, c_i32),
    "moe_dispatch_reroute": ([_SP] + [c_p] * 15 + [c_size, c_p], c_i32),
    "moe_dispatch_fp8": ([_SP] + [c_p] * 15 + [c_size, c_p], c_i32),
    "moe_quantize_rows_e4m3": ([c_p, c_i64, c_i32, c_p, c_p, c_p, c_p], c_i32),
    "moe_convert_bf16_to_f16": ([c_p, c_i64, c_p, c_p, c_p], c_i32),
    "moe_expert_up_fp8": ([_SP] + [c_p] * 9, c_i32),
    "moe_expert_down_fp8": ([_SP] + [c_p] * 7, c_i32),
    "moe_layer_fp8": ([_SP] + [c_p] * 14 + [c_size, c_p], c_i32),
    "moe_expert_gemm": ([_SP] + [c_p] * 8, c_i32),
    "moe_expert_up": ([_SP] + [c_p] * 6, c_i32),
    "moe_expert_down": ([_SP] + [c_p] * 5, c_i32),
    "moe_combine": ([_SP] + [c_p] * 7, c_i32),
    "moe_shared_expert": ([_SP, c_i32] + [c_p] * 7 + [c_size, c_p], c_i32),
    "moe_layer_shared_workspace_size": ([_SP, c_i32], c_size),
    "moe_layer_shared": ([_SP, c_i32] + [c_p] * 14 + [c_size, c_p], c_i32),
    "moe_layer": ([_SP] + [c_p] * 11 + [c_size, c_p], c_i32),
    "moe_affinity_accumulate": ([c_i32, c_i32, c_i32, c_p, c_p, c_p, c_p], c_i32),
    "moe_derive_report": ([_SP, ctypes.POINTER(MoeStats), c_p, c_p, ctypes.POINTER(MoeReport)],
                          c_i32),
    "moe_exchange_schedule": ([c_i32, c_p, c_i32, c_p, c_p, c_p, c_p], c_i32),
    "moe_place_experts": ([c_i32, c_i32, c_i32, c_p, c_i32, c_p, c_p, c_p], c_i32),
    "moe_place_experts_staged": ([c_i32] * 4 + [c_p, c_i32] + [c_p] * 5, c_i32),
    "moe_placement_order": ([c_i32] * 3 + [c_p] * 2, c_i32),
    "moe_get_device_error": ([ctypes.c_int], c_i32),
    "moe_read_stats": ([c_p, ctypes.POINTER(MoeStats), c_p], c_i32),
    "moe_debug_bounded_wait": ([c_u64, c_p], c_i32),
}


ABI_VERSION = 3  # MOE_ABI_VERSION the structures below match


class _Lib:
    """Loads libmoe_b200.so on first use and declares every C signature."""

    def __init__(self):
        self._cdll = None

    def _load(self):
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m combine_grouped_gemm_router_b200.build` (nvcc, sm_100a). "
                "There is no CPU fallback.")
        cdll = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _sigs.items():
            fn = getattr(cdll, name)
            fn.argtypes = args
            fn.restype = res
        if cdll.moe_abi_version() != ABI_VERSION:
            raise ImportError(f"{LIB_PATH} has ABI version {cdll.moe_abi_version()}, this binding "
                              f"expects {ABI_VERSION}: rebuild it")
        self._cdll = cdll

    def __getattr__(self, name):
        if self._cdll is None:
            self._load()
        return getattr(self._cdll, name)


_lib = _Lib()


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


def _check(rc: int, where: str) -> None:
    if rc != MOE_OK:
        raise MoeError(rc, where)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


MOE_FLAG_OUT_BF16 = 1
MOE_FLAG_SLOT_MAJOR = 2
MOE_FLAG_REROUTE = 4
MOE_FLAG_FP8_RETURN = 8
MOE_FLAG_H_BF16 = 16
MOE_FLAG_Y_F16 = 32


def make_shape(N: int, d: int, f: int, E: int, K: int, W: int, capacity_factor: float = 0.0,
               out_bf16: bool = False, slot_major: bool = False,
               reroute: bool = False, fp8_return: bool = False, h_bf16: bool = False,
               y_f16: bool = False) -> MoeShape:
    """h_bf16: the SwiGLU activation h and the down-projection weights in bf16 instead of the
    default fp16 (then W2 is passed as the bf16 weights, not their fp16 copy)."""
    flags = ((MOE_FLAG_OUT_BF16 if out_bf16 else 0) | (MOE_FLAG_SLOT_MAJOR if slot_major else 0)
             | (MOE_FLAG_REROUTE if reroute else 0) | (MOE_FLAG_FP8_RETURN if fp8_return else 0)
             | (MOE_FLAG_H_BF16 if h_bf16 else 0) | (MOE_FLAG_Y_F16 if y_f16 else 0))
    return MoeShape(N, d, f, E, K, W, float(capacity_factor), flags)


# ---------------------------------------------------------------- sizes

def moe_abi_version() -> int:
    return _lib.moe_abi_version()


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def moe_capacity(shape: MoeShape) -> int:
    return _lib.moe_capacity(ctypes.byref(shape))


def moe_y_bytes(shape: MoeShape) -> int:
    """Bytes of the expert-output buffer y (fp32 rows, or the FP8 return payload)."""
    return _lib.moe_y_bytes(ctypes.byref(shape))


def y_payload_stride(shape: MoeShape) -> int:
    """Row stride in bytes of the y payload: d e4m3 codes (FP8 return) or 2d bytes of fp16 codes
    (MOE_FLAG_Y_F16), then d/32 exponents, padded to 16."""
    codes = 2 * shape.d if shape.flags & MOE_FLAG_Y_F16 else shape.d
    return codes + ((shape.d // 32 + 15) // 16) * 16


def moe_rows_alloc(shape: MoeShape) -> int:
    return _lib.moe_rows_alloc(ctypes.byref(shape))


def moe_workspace_size(shape: MoeShape) -> int:
    return _lib.moe_workspace_size(ctypes.byref(shape))


def moe_layer_workspace_size(shape: MoeShape) -> int:
    return _lib.moe_layer_workspace_size(ctypes.byref(shape))


# ---------------------------------------------------------------- stages

def moe_route(shape, x, w_router, bias, topk_idx, topk_w, logits=None, ws=None, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_route(ctypes.byref(shape), _ptr(x), _ptr(w_router), _ptr(bias),
                          _ptr(topk_idx), _ptr(topk_w), _ptr(logits), _ptr(ws), ws_bytes,
                          _stream(stream)), "moe_route")


def moe_dispatch(shape, x, topk_idx, counts, kept, offsets, row_of, assign_of_row, x_sorted,
                 x_packed=None, rank_matrix=None, packed_offsets=None, stats=None, ws=None,
                 stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_dispatch(ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(counts),
                             _ptr(kept), _ptr(offsets), _ptr(row_of), _ptr(assign_of_row),
                             _ptr(x_sorted), _ptr(x_packed), _ptr(rank_matrix),
                             _ptr(packed_offsets), _ptr(stats), _ptr(ws), ws_bytes,
                             _stream(stream)), "moe_dispatch")


def moe_dispatch_rank(shape, rank, x_local, topk_idx_all, counts, kept, offsets, row_of,
                      assign_of_row, packed_row_of, send_row_of, x_send, rank_matrix,
                      packed_offsets, stats=None, ws=None, stream=None):
    """Rank `rank`'s dispatch with W real ranks (shape: the whole batch)."""
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_dispatch_rank(ctypes.byref(shape), int(rank), _ptr(x_local),
                                  _ptr(topk_idx_all), _ptr(counts), _ptr(kept), _ptr(offsets),
                                  _ptr(row_of), _ptr(assign_of_row), _ptr(packed_row_of),
                                  _ptr(send_row_of), _ptr(x_send), _ptr(rank_matrix),
                                  _ptr(packed_offsets), _ptr(stats), _ptr(ws), ws_bytes,
                                  _stream(stream)), "moe_dispatch_rank")


def moe_regroup_rows(shape, rank, direction, src, dst, assign_of_row, packed_row_of, offsets,
                     packed_offsets, offsets_local=None, row_bytes=None, stream=None):
    """Rows of rank `rank` between the exchange's order (direction 0: src) and its experts'
    order (direction 1: src). row_bytes defaults to the byte size of one row of src."""
    if row_bytes is None:
        row_bytes = src[0].numel() * src.element_size() if src.dim() > 1 else src.element_size()
    _check(_lib.moe_regroup_rows(ctypes.byref(shape), int(rank), int(row_bytes), int(direction),
                                 _ptr(src), _ptr(dst), _ptr(assign_of_row), _ptr(packed_row_of),
                                 _ptr(offsets), _ptr(packed_offsets), _ptr(offsets_local),
                                 _stream(stream)), "moe_regroup_rows")


def moe_dispatch_reroute(shape, x, logits, topk_idx, counts, kept, offsets, row_of,
                         assign_of_row, x_sorted, expert_of=None, x_packed=None,
                         rank_matrix=None, packed_offsets=None, stats=None, ws=None, stream=None):
    """moe_dispatch with overflowed assignments moved to the next-best non-full expert
    (shape made with reroute=True; logits as written by moe_route)."""
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_dispatch_reroute(ctypes.byref(shape), _ptr(x), _ptr(logits), _ptr(topk_idx),
                                     _ptr(counts), _ptr(kept), _ptr(offsets), _ptr(row_of),
                                     _ptr(assign_of_row), _ptr(expert_of), _ptr(x_sorted),
                                     _ptr(x_packed), _ptr(rank_matrix), _ptr(packed_offsets),
                                     _ptr(stats), _ptr(ws), ws_bytes, _stream(stream)),
           "moe_dispatch_reroute")


def moe_dispatch_fp8(shape, x, topk_idx, counts, kept, offsets, row_of, assign_of_row, x_sorted,
                     sorted_scale, x_packed=None, packed_scale=None, rank_matrix=None,
                     packed_offsets=None, stats=None, ws=None, stream=None):
    """moe_dispatch writing the FP8 payload: e4m3 rows (uint8) with one scale per row."""
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_dispatch_fp8(ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(counts),
                                 _ptr(kept), _ptr(offsets), _ptr(row_of), _ptr(assign_of_row),
                                 _ptr(x_sorted), _ptr(sorted_scale), _ptr(x_packed),
                                 _ptr(packed_scale), _ptr(rank_matrix), _ptr(packed_offsets),
                                 _ptr(stats), _ptr(ws), ws_bytes, _stream(stream)),
           "moe_dispatch_fp8")


def moe_quantize_rows_e4m3(src, codes, scale, rows_dev=None, stream=None):
    """Row-wise e4m3 quantisation of a bf16 matrix (rows = all leading dims); rows_dev
    (optional device int32 tensor) caps the row count on the device."""
    cols = src.shape[-1]
    rows = src.numel() // cols
    _check(_lib.moe_quantize_rows_e4m3(_ptr(src), rows, cols, _ptr(codes), _ptr(scale),
                                       _ptr(rows_dev), _stream(stream)), "moe_quantize_rows_e4m3")


def moe_convert_bf16_to_f16(src, dst, changed=None, stream=None):
    """fp16 copy of a bf16 weight array (all elements; the down projection's W2 / Ws2);
    changed (optional device int64 tensor of one element) accumulates the count of elements
    whose value changed."""
    n = src.numel()
    if dst.numel() != n:
        raise MoeError(1, "moe_convert_bf16_to_f16: src and dst sizes differ")
    _check(_lib.moe_convert_bf16_to_f16(_ptr(src), n, _ptr(dst), _ptr(changed), _stream(stream)),
           "moe_convert_bf16_to_f16")


def w2_for(shape, w2, stream=None):
    """The down-projection weights in the form `shape` asks for: the bf16 tensor itself with
    h_bf16, else a new fp16 copy made by moe_convert_bf16_to_f16."""
    if shape.flags & MOE_FLAG_H_BF16:
        return w2
    import torch
    out = torch.empty(w2.shape, dtype=torch.float16, device=w2.device)
    moe_convert_bf16_to_f16(w2, out, stream=stream)
    return out


def moe_expert_up_fp8(shape, x_sorted, sorted_scale, offsets, w1q, w1_scale, w3q, w3_scale, h,
                      stream=None):
    _check(_lib.moe_expert_up_fp8(ctypes.byref(shape), _ptr(x_sorted), _ptr(sorted_scale),
                                  _ptr(offsets), _ptr(w1q), _ptr(w1_scale), _ptr(w3q),
                                  _ptr(w3_scale), _ptr(h), _stream(stream)), "moe_expert_up_fp8")


def moe_expert_down_fp8(shape, hq, h_scale, offsets, w2q, w2_scale, y, stream=None):
    _check(_lib.moe_expert_down_fp8(ctypes.byref(shape), _ptr(hq), _ptr(h_scale), _ptr(offsets),
                                    _ptr(w2q), _ptr(w2_scale), _ptr(y), _stream(stream)),
           "moe_expert_down_fp8")


MOE_STATIC_SCRATCH_BYTES = 1 << 20


def moe_dispatch_static(shape, x, topk_idx, counts, kept, offsets, row_of, assign_of_row,
                        x_sorted, x_packed=None, rank_matrix=None, packed_offsets=None, stats=None,
                        stream=None):
    """moe_dispatch with the library's fixed device scratch instead of a caller workspace
    (for callers that cannot allocate device memory)."""
    _check(_lib.moe_dispatch_static(ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(counts),
                                    _ptr(kept), _ptr(offsets), _ptr(row_of), _ptr(assign_of_row),
                                    _ptr(x_sorted), _ptr(x_packed), _ptr(rank_matrix),
                                    _ptr(packed_offsets), _ptr(stats), _stream(stream)),
           "moe_dispatch_static")


def moe_expert_gemm(shape, x_sorted, offsets, w1, w3, w2, h, y, stream=None):
    _check(_lib.moe_expert_gemm(ctypes.byref(shape), _ptr(x_sorted), _ptr(offsets), _ptr(w1),
                                _ptr(w3), _ptr(w2), _ptr(h), _ptr(y), _stream(stream)),
           "moe_expert_gemm")


def moe_expert_up(shape, x_sorted, offsets, w1, w3, h, stream=None):
    _check(_lib.moe_expert_up(ctypes.byref(shape), _ptr(x_sorted), _ptr(offsets), _ptr(w1),
                              _ptr(w3), _ptr(h), _stream(stream)), "moe_expert_up")


def moe_expert_down(shape, h, offsets, w2, y, stream=None):
    _check(_lib.moe_expert_down(ctypes.byref(shape), _ptr(h), _ptr(offsets), _ptr(w2), _ptr(y),
                                _stream(stream)), "moe_expert_down")


def moe_combine(shape, y, row_of, topk_w, out, residual=None, shared_y=None, stream=None):
    _check(_lib.moe_combine(ctypes.byref(shape), _ptr(y), _ptr(row_of), _ptr(topk_w),
                            _ptr(shared_y), _ptr(residual), _ptr(out), _stream(stream)),
           "moe_combine")


def moe_shared_expert(shape, f_shared, x, ws1, ws3, ws2, h_s, y_s, ws, stream=None):
    _check(_lib.moe_shared_expert(ctypes.byref(shape), int(f_shared), _ptr(x), _ptr(ws1),
                                  _ptr(ws3), _ptr(ws2), _ptr(h_s), _ptr(y_s), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)),
           "moe_shared_expert")


def moe_layer_shared_workspace_size(shape, f_shared) -> int:
    return _lib.moe_layer_shared_workspace_size(ctypes.byref(shape), int(f_shared))


def moe_layer_shared(shape, f_shared, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, out,
                     residual=None, topk_idx_out=None, stats=None, ws=None, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_layer_shared(ctypes.byref(shape), int(f_shared), _ptr(x), _ptr(w_router),
                                 _ptr(bias), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(ws1), _ptr(ws3),
                                 _ptr(ws2), _ptr(residual), _ptr(out), _ptr(topk_idx_out),
                                 _ptr(stats), _ptr(ws), ws_bytes, _stream(stream)),
           "moe_layer_shared")


def moe_layer(shape, x, w_router, bias, w1, w3, w2, out, residual=None, topk_idx_out=None,
              stats=None, ws=None, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_layer(ctypes.byref(shape), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w1),
                          _ptr(w3), _ptr(w2), _ptr(residual), _ptr(out), _ptr(topk_idx_out),
                          _ptr(stats), _ptr(ws), ws_bytes, _stream(stream)), "moe_layer")


def moe_layer_fp8(shape, x, w_router, bias, w1q, w1_scale, w3q, w3_scale, w2q, w2_scale, out,
                  residual=None, topk_idx_out=None, stats=None, ws=None, stream=None):
    """moe_layer with the FP8 payload and e4m3 expert GEMMs (weights from
    moe_quantize_rows_e4m3)."""
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_layer_fp8(ctypes.byref(shape), _ptr(x), _ptr(w_router), _ptr(bias),
                              _ptr(w1q), _ptr(w1_scale), _ptr(w3q), _ptr(w3_scale), _ptr(w2q),
                              _ptr(w2_scale), _ptr(residual), _ptr(out), _ptr(topk_idx_out),
                              _ptr(stats), _ptr(ws), ws_bytes, _stream(stream)), "moe_layer_fp8")


def moe_affinity_accumulate(N, E, K, topk_j, topk_j1, counts, stream=None):
    _check(_lib.moe_affinity_accumulate(N, E, K, _ptr(topk_j), _ptr(topk_j1), _ptr(counts),
                                        _stream(stream)), "moe_affinity_accumulate")


# ---------------------------------------------------------------- host helpers

def moe_derive_report(shape, stats: MoeStats, rank_matrix, kept) -> MoeReport:
    """rank_matrix: host int64 [W*W] array-like; kept: host int32 [E]."""
    import numpy as np
    D = np.ascontiguousarray(rank_matrix, dtype=np.int64).reshape(-1)
    k = np.ascontiguousarray(kept, dtype=np.int32).reshape(-1)
    rep = MoeReport()
    _check(_lib.moe_derive_report(ctypes.byref(shape), ctypes.byref(stats),
                                  D.ctypes.data_as(c_p), k.ctypes.data_as(c_p),
                                  ctypes.byref(rep)), "moe_derive_report")
    return rep


def moe_exchange_schedule(rank_matrix, max_phases: Optional[int] = None):
    """Contention-free transmission order of one exchange (host arrays in, host arrays out).

    rank_matrix: int64 [W, W]. Returns (phase_dst int32 [n, W], phase_len int64 [n], makespan).
    """
    import numpy as np
    D = np.ascontiguousarray(rank_matrix, dtype=np.int64)
    W = int(round(D.size ** 0.5))
    if D.size != W * W:
        raise MoeError(1, "moe_exchange_schedule: rank_matrix is not square")
    cap = 2 * W * W if max_phases is None else int(max_phases)
    dst = np.empty((max(cap, 1), W), np.int32)
    ln = np.empty(max(cap, 1), np.int64)
    n = ctypes.c_int32(0)
    span = ctypes.c_int64(0)
    _check(_lib.moe_exchange_schedule(W, D.ctypes.data_as(c_p), cap, dst.ctypes.data_as(c_p),
                                      ln.ctypes.data_as(c_p), ctypes.byref(n),
                                      ctypes.byref(span)), "moe_exchange_schedule")
    return dst[:n.value].copy(), ln[:n.value].copy(), int(span.value)


def moe_place_experts(counts, L: int, E: int, P: int, starts: int = 16):
    """Expert placement from affinity counts int64 [L-1, E, E] (host).

    Returns (gpu_of int32 [L, E], cost, contiguous_cost).
    """
    import numpy as np
    c = np.ascontiguousarray(counts, dtype=np.int64).reshape(-1)
    if c.size != max(L - 1, 0) * E * E:
        raise MoeError(1, "moe_place_experts: counts must hold (L-1)*E*E entries")
    g = np.empty((L, E), np.int32)
    cost = ctypes.c_int64(0)
    base = ctypes.c_int64(0)
    _check(_lib.moe_place_experts(int(L), int(E), int(P),
                                  c.ctypes.data_as(c_p) if c.size else None, int(starts),
                                  g.ctypes.data_as(c_p), ctypes.byref(cost), ctypes.byref(base)),
           "moe_place_experts")
    return g, int(cost.value), int(base.value)


def placement_order(gpu_of, P: int):
    """Storage order that deploys a placement (moe_placement_order): order[l][s] = the expert of
    layer l to store at slot s, GPU by GPU; permute the router rows and expert weights with it."""
    import numpy as np
    g = np.ascontiguousarray(gpu_of, dtype=np.int32)
    L, E = g.shape
    order = np.empty((L, E), np.int32)
    _check(_lib.moe_placement_order(L, E, int(P), g.ctypes.data_as(c_p),
                                    order.ctypes.data_as(c_p)), "moe_placement_order")
    return order


def moe_place_experts_staged(counts, L: int, E: int, nodes: int, gpus_per_node: int,
                             starts: int = 16):
    """Two-stage placement (nodes, then GPUs inside each node) from affinity counts
    int64 [L-1, E, E]. Returns (gpu_of int32 [L, E], dict of node/GPU hop counts, placed and
    contiguous)."""
    import numpy as np
    c = np.ascontiguousarray(counts, dtype=np.int64).reshape(-1)
    if c.size != max(L - 1, 0) * E * E:
        raise MoeError(1, "moe_place_experts_staged: counts must hold (L-1)*E*E entries")
    g = np.empty((L, E), np.int32)
    out = [ctypes.c_int64(0) for _ in range(4)]
    _check(_lib.moe_place_experts_staged(int(L), int(E), int(nodes), int(gpus_per_node),
                                         c.ctypes.data_as(c_p) if c.size else None, int(starts),
                                         g.ctypes.data_as(c_p),
                                         *[ctypes.byref(v) for v in out]),
           "moe_place_experts_staged")
    keys = ("node_hops", "gpu_hops", "contiguous_node_hops", "contiguous_gpu_hops")
    return g, {k: int(v.value) for k, v in zip(keys, out)}


def moe_get_device_error(clear: bool = True) -> int:
    """Status recorded by kernels on the current device (synchronises)."""
    return _lib.moe_get_device_error(1 if clear else 0)


def moe_debug_bounded_wait(timeout_ns: int, stream=None) -> None:
    _check(_lib.moe_debug_bounded_wait(int(timeout_ns), _stream(stream)), "moe_debug_bounded_wait")


def stats_buffer(device="cuda"):
    """A device buffer of sizeof(moe_stats_t) bytes."""
    import torch
    return torch.zeros(ctypes.sizeof(MoeStats), dtype=torch.uint8, device=device)


def read_stats(buf, stream=None) -> MoeStats:
    """The counters in a device stats buffer, through moe_read_stats (waits for the stream)."""
    st = MoeStats()
    _check(_lib.moe_read_stats(_ptr(buf), ctypes.byref(st), _stream(stream)), "moe_read_stats")
    return st


def report_dict(rep: MoeReport) -> dict:
    return {name: getattr(rep, name) for name, _ in MoeReport._fields_}


def stats_dict(st: MoeStats) -> dict:
    return {name: getattr(st, name) for name, _ in MoeStats._fields_}
