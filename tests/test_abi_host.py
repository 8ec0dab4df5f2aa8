"""The C-ABI library on the CPU: it loads, exports every symbol the header
declares, validates arguments before launching anything, and its host-side
report agrees with the oracle's definitions. No compute call needs a GPU here:
every call below returns before any CUDA API is reached."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def m():
    from combine_grouped_gemm_router_b200 import build
    build.build()
    import combine_grouped_gemm_router_b200 as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(m):
    lib = ctypes.CDLL(m.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 14, names
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version_and_status_strings(m):
    assert m.moe_abi_version() == 3
    for code, name in m.STATUS_NAMES.items():
        assert m.moe_status_string(code) == name
    assert m.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def test_capacity_and_rows_alloc_match_oracle(m, orc):
    cases = [(8192, 2048, 768, 128, 8, 8, 1.25), (32768, 4096, 1536, 64, 6, 8, 1.0),
             (32768, 4096, 1536, 64, 6, 8, 2.0), (4096, 4096, 14336, 8, 2, 8, 0.0),
             (16, 7168, 2048, 256, 8, 8, 0.0), (10, 8, 128, 5, 2, 5, 0.7)]
    for N, d, f, E, K, W, cf in cases:
        s = m.make_shape(N, d, f, E, K, W, cf)
        C = orc.capacity(N, E, K, cf)
        assert m.moe_capacity(s) == C
        assert m.moe_rows_alloc(s) == min(N * K, E * min(C, N * K)) + 128


def test_shape_validation(m):
    ok = m.make_shape(64, 128, 256, 8, 2, 4, 0.0)
    assert m.moe_workspace_size(ok) > 0 and m.moe_layer_workspace_size(ok) > 0
    bad = [m.make_shape(64, 128, 256, 8, 9, 4),      # K > E
           m.make_shape(64, 128, 256, 8, 2, 3),      # E % W
           m.make_shape(66, 128, 256, 8, 2, 4),      # N % W
           m.make_shape(-4, 128, 256, 8, 2, 4),      # N < 0
           m.make_shape(64, 100, 256, 8, 2, 4),      # d % 8
           m.make_shape(64, 128, 256, 512, 2, 4),    # E > 256
           m.make_shape(64, 128, 256, 64, 33, 4)]    # K > 32
    for s in bad:
        assert m.moe_rows_alloc(s) == -1
        assert m.moe_workspace_size(s) == 0
    flags = m.make_shape(64, 128, 256, 8, 2, 4)
    flags.flags = 1 << 10  # no such flag
    assert m.moe_workspace_size(flags) == 0
    # an empty batch is a valid shape
    assert m.moe_workspace_size(m.make_shape(0, 128, 256, 8, 2, 4)) > 0
    assert m.moe_rows_alloc(m.make_shape(0, 128, 256, 8, 2, 4)) == 128
    assert m.moe_workspace_size(m.make_shape(64, 128, 256, 8, 2, 4, out_bf16=True)) > 0
    # slot-major priority scans K blocks per token block: a larger scratch, never smaller
    tm = m.moe_workspace_size(m.make_shape(4096, 128, 256, 256, 32, 64, 1.0))
    sm = m.moe_workspace_size(m.make_shape(4096, 128, 256, 256, 32, 64, 1.0, slot_major=True))
    assert 0 < tm < sm
    # GEMM shapes: d % 128, f % 128
    assert m.moe_layer_workspace_size(m.make_shape(64, 136, 256, 8, 2, 4)) == 0
    assert m.moe_layer_workspace_size(m.make_shape(64, 128, 200, 8, 2, 4)) == 0


def _raw(m):
    return m._lib


def test_argument_errors_return_before_launch(m):
    lib = _raw(m)
    s = m.make_shape(64, 128, 256, 8, 2, 4, 0.0)
    P = 0x100000  # a fake, 16-byte aligned address: never dereferenced
    by = ctypes.byref
    # null pointers
    assert lib.moe_route(by(s), None, P, None, P, P, P, None, 0, None) == 1
    assert lib.moe_expert_gemm(by(s), P, P, P, P, None, P, P, None) == 1
    assert lib.moe_combine(by(s), P, P, P, None, None, None, None) == 1
    # misaligned
    assert lib.moe_route(by(s), P + 2, P, None, P, P, P, None, 0, None) == 4
    assert lib.moe_combine(by(s), P + 8, P, P, None, None, P, None) == 4
    assert lib.moe_combine(by(s), P, P, P, P + 4, None, P, None) == 4  # misaligned shared_y
    assert lib.moe_shared_expert(by(s), 100, P, P, P, P, P, P, P, 256, None) == 2
    assert lib.moe_shared_expert(by(s), 128, P, P, P, P, P, P, P, 16, None) == 3
    assert m.moe_layer_shared_workspace_size(s, 100) == 0
    assert m.moe_layer_shared_workspace_size(s, 256) > m.moe_layer_workspace_size(s)
    # workspace too small (logits requested in the workspace)
    assert lib.moe_route(by(s), P, P, None, P, P, None, P, 16, None) == 3
    need = m.moe_workspace_size(s)
    assert lib.moe_dispatch(by(s), P, P, P, P, P, P, P, P, None, None, None, None, P, need - 1,
                            None) == 3
    assert lib.moe_layer(by(s), P, P, None, P, P, P, None, P, None, None, P, 1024, None) == 3
    # the fused router (N >= 2048, E > 32) reads the router weights transposed into the
    # workspace: required even when the logits go to the caller, and sized for [d][E rounded up]
    big = m.make_shape(4096, 7168, 256, 200, 8, 8)
    assert lib.moe_route(by(big), P, P, None, P, P, P, None, 0, None) == 3
    assert lib.moe_route(by(big), P, P, None, P, P, P, P, 16, None) == 3
    assert m.moe_workspace_size(big) >= 256 * 7168 * 4 > 4096 * 200 * 4
    few = m.make_shape(2047, 7168, 256, 200, 8, 1)  # the two-kernel router: no workspace needed
    assert m.moe_workspace_size(few) < 256 * 7168 * 4
    # shape errors
    bad = m.make_shape(64, 128, 256, 8, 9, 4)
    assert lib.moe_route(by(bad), P, P, None, P, P, P, None, 0, None) == 1
    assert lib.moe_expert_gemm(by(m.make_shape(64, 192, 256, 8, 2, 4)), P, P, P, P, P, P, P,
                               None) == 2
    # re-routing needs the logits: refused by the entry points that do not take them
    rr = m.make_shape(64, 128, 256, 8, 2, 4, 1.0, reroute=True)
    need_rr = m.moe_workspace_size(rr)
    assert need_rr > need  # the moved-expert array
    assert lib.moe_dispatch(by(rr), P, P, P, P, P, P, P, P, None, None, None, None, P, need_rr,
                            None) == 1
    assert lib.moe_dispatch_static(by(rr), P, P, P, P, P, P, P, P, None, None, None, None,
                                   None) == 1
    assert lib.moe_dispatch_reroute(by(rr), P, None, P, P, P, P, P, P, None, P, None, None, None,
                                    None, P, need_rr, None) == 1  # no logits
    assert lib.moe_dispatch_reroute(by(s), P, P, P, P, P, P, P, P, None, P, None, None, None,
                                    None, P, need, None) == 1  # flag not set
    assert lib.moe_dispatch_reroute(by(rr), P, P + 2, P, P, P, P, P, P, None, P, None, None, None,
                                    None, P, need_rr, None) == 4  # misaligned logits
    assert lib.moe_dispatch_reroute(by(rr), P, P, P, P, P, P, P, P, None, P, None, None, None,
                                    None, P, need_rr - 1, None) == 3
    # FP8 payload entry points
    assert lib.moe_dispatch_fp8(by(s), P, P, P, P, P, P, P, P, None, None, None, None, None, None,
                                P, need, None) == 1  # no row scales
    assert lib.moe_dispatch_fp8(by(s), P, P, P, P, P, P, P, P, P, P, None, None, None, None, P,
                                need, None) == 1  # packed rows without packed scales
    assert lib.moe_dispatch_fp8(by(s), P, P, P, P, P, P, P, P, P + 2, None, None, None, None,
                                None, P, need, None) == 4  # misaligned scale
    assert lib.moe_dispatch_fp8(by(rr), P, P, P, P, P, P, P, P, P, None, None, None, None, None,
                                P, need_rr, None) == 1  # re-routing needs the logits
    assert lib.moe_quantize_rows_e4m3(P, 4, 24, P, P, None, None) == 2  # cols % 16
    assert lib.moe_quantize_rows_e4m3(P, 4, 32, P + 8, P, None, None) == 4
    assert lib.moe_quantize_rows_e4m3(P, 4, 32, P, P, P + 2, None) == 4  # row count alignment
    assert lib.moe_quantize_rows_e4m3(None, 4, 32, P, P, None, None) == 1
    assert lib.moe_quantize_rows_e4m3(P, 0, 32, P, P, None, None) == 0  # nothing to do
    assert lib.moe_expert_down_fp8(by(s), P, None, P, P, P, P, None) == 1
    assert lib.moe_expert_down_fp8(by(s), P, P, P, P, P + 4, P, None) == 4
    assert lib.moe_expert_up_fp8(by(s), P, P, P, P, P + 4, P, P, P, None) == 4  # scale alignment
    assert lib.moe_expert_up_fp8(by(s), P, None, P, P, P, P, P, P, None) == 1
    assert lib.moe_layer_fp8(by(s), P, P, None, P, P, P, P, P, P, None, P, None, None, P, 1024,
                             None) == 3
    assert lib.moe_layer_fp8(by(s), P, P, None, P, P, P, P, P, None, None, P, None, None, P,
                             1 << 30, None) == 1  # no W2 scales
    assert lib.moe_affinity_accumulate(10, 8, 9, P, P, P, None) == 1
    assert lib.moe_affinity_accumulate(10, 300, 2, P, P, P, None) == 2
    assert lib.moe_debug_bounded_wait(0, None) == 1
    # the fp16 copy of the down-projection weights
    assert lib.moe_convert_bf16_to_f16(P, 12, P, None, None) == 2   # n % 8
    assert lib.moe_convert_bf16_to_f16(None, 16, P, None, None) == 1
    assert lib.moe_convert_bf16_to_f16(P, -8, P, None, None) == 1
    assert lib.moe_convert_bf16_to_f16(P + 2, 16, P, None, None) == 4
    assert lib.moe_convert_bf16_to_f16(P, 16, P, P + 4, None) == 4   # counter alignment
    assert lib.moe_convert_bf16_to_f16(None, 0, None, None, None) == 0  # nothing to do
    assert m.moe_status_string(9) == "MOE_ERR_F16_RANGE"
    # every flag bit the header defines is accepted; the bf16 h flag among them
    assert m.moe_layer_workspace_size(m.make_shape(64, 128, 256, 8, 2, 4, h_bf16=True)) == \
        m.moe_layer_workspace_size(s)


def test_derive_report_matches_oracle(m, orc):
    import json
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "hand_routing.json")))
    s = m.make_shape(g["N"], 8, 128, g["E"], g["K"], g["W"], g["cf"])
    st = m.MoeStats(rows=7, dropped=1, cross_rows=2, dedup_pairs=2, nonfinite_tokens=0,
                    capacity=2, active_experts=4, max_kept=2, min_kept=1)
    rep = m.report_dict(m.moe_derive_report(s, st, np.array(g["D"]).reshape(-1), g["kept"]))
    for k, v in g["report"].items():
        assert rep[k] == pytest.approx(v, rel=1e-12), k
    # random routings: every derived figure equals the oracle's
    rng = np.random.default_rng(1)
    for trial in range(5):
        N, E, K, W = 512, 32, 4, 8
        lg = rng.standard_normal((N, E)).astype(np.float32)
        lg += np.array([-1.1 * math.log(e + 1) for e in range(E)], np.float32) * (trial % 2)
        idx, _, _ = orc.topk(lg, K)
        cf = [0.0, 1.0, 1.25, 0.5, 2.0][trial]
        C = orc.capacity(N, E, K, cf)
        p = orc.positions(idx, E, W, C)
        ref = orc.derive_report(N, E, K, W, p["kept"], p["D"], p["stats"], d=256)
        ps = p["stats"]
        st = m.MoeStats(rows=ps["R"], dropped=ps["dropped"], cross_rows=ps["cross_rows"],
                        dedup_pairs=ps["dedup_pairs"], nonfinite_tokens=0,
                        capacity=min(C, N * K), active_experts=ps["active_experts"],
                        max_kept=ps["max_kept"], min_kept=ps["min_kept"])
        rep = m.report_dict(m.moe_derive_report(m.make_shape(N, 256, 128, E, K, W, cf), st,
                                                p["D"].reshape(-1), p["kept"]))
        for k in ("drop_rate", "send_max_over_min", "recv_max_over_min", "cross_rank_fraction",
                  "load_std_over_mean", "capacity_factor_effective", "tau_min_tokens",
                  "dispatch_bytes", "send_max", "send_min", "recv_max", "recv_min"):
            assert rep[k] == pytest.approx(ref[k], rel=1e-12), (trial, k)


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib
    import combine_grouped_gemm_router_b200 as mod
    fresh = mod._Lib()
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        fresh.moe_abi_version()
    importlib.reload(mod)


def test_graft_build_entry():
    """The build entry point compiles (or finds current) the library and the oracle and checks
    the library's ABI version against the binding's."""
    import __graft_entry__
    __graft_entry__.build()


def test_y_buffer_sizes(m):
    """fp32 y: rows_alloc * d * 4 bytes; the FP8 return payload: rows_alloc rows of d codes
    plus d/32 exponent bytes padded to 16 (d = 128: 4 -> 16; 2048: 64; 7168: 224)."""
    for d, pad in ((128, 16), (384, 16), (2048, 64), (7168, 224)):
        s = m.make_shape(64, d, 256, 8, 2, 4)
        s8 = m.make_shape(64, d, 256, 8, 2, 4, fp8_return=True)
        RA = m.moe_rows_alloc(s)
        assert m.moe_y_bytes(s) == RA * d * 4
        assert m.y_payload_stride(s8) == d + pad and (d + pad) % 16 == 0
        assert m.moe_y_bytes(s8) == RA * (d + pad)
    # the payload needs d % 128 == 0 (the down GEMM's tiles), also for the combine alone
    assert m.moe_y_bytes(m.make_shape(64, 136, 256, 8, 2, 4, fp8_return=True)) == 0
    P = 0x100000  # a fake, 16-byte aligned address: never dereferenced
    s8 = m.make_shape(64, 136, 256, 8, 2, 4, fp8_return=True)
    assert _raw(m).moe_combine(ctypes.byref(s8), P, P, P, None, None, P, None) == 2


def test_header_is_plain_c(tmp_path):
    """include/moe_b200.h is a C header: it compiles as strict C11 (no C++ or CUDA types in the
    signatures), and a C program can call a host entry point through it and link."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use.c"
    src.write_text(
        '#include "moe_b200.h"\n'
        "int main(void) {\n"
        "    moe_shape_t s = {64, 128, 256, 8, 2, 4, 0.0f, 0u};\n"
        "    return moe_capacity(&s) == 128 && moe_abi_version() == MOE_ABI_VERSION ? 0 : 1;\n"
        "}\n")
    lib_dir = os.path.join(root, "combine_grouped_gemm_router_b200")
    exe = tmp_path / "use"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(root, "include"), str(src), "-o", str(exe),
                    "-L", lib_dir, "-l:libmoe_b200.so", "-Wl,-rpath," + lib_dir],
                   check=True, capture_output=True)
    assert subprocess.run([str(exe)]).returncode == 0
