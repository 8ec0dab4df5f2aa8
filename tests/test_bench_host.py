"""Host-side checks of the benchmark harness: the launch count it claims per workload (the
library's launch rules, each count also seen in an ncu launch list of that workload), and the
reference arm's JSON line (the oracle timed on the host cores) on the smallest workload."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


@pytest.mark.parametrize("name,count", [
    ("mixtral_prefill", 10),       # E = 8: projection, then selection; pair + single GEMMs,
                                   # the fp16 range pass
    ("mixtral_prefill_fp8", 10),   # e4m3 GEMMs (no range pass) + quantisation of h
    ("e128_skew", 8),              # W_r transposition + fused router; ~165 rows per expert:
                                   # single-CTA GEMMs only
    ("e128_skew_fp8", 8),
    ("decode", 8),                 # 16 tokens: projection, then selection
    ("e128_skew_slot_major", 8),   # the same two dispatch kernels over K times more blocks
    ("e128_skew_reroute", 11),     # positions-only pass, the ranking kernel, the full pass
    ("stack4", 10),                # pair GEMMs
    ("stack4_affinity", 10),
    ("mixtral_prefill_fp8_return", 10),
    ("e128_skew_fp8_return", 8),
    ("residual_top1", 14),         # shared MLP: offsets, pair + single GEMMs twice, range passes
])
def test_kernel_launch_count(name, count):
    import bench
    from moe_workloads import WORKLOADS
    assert bench.kernel_launches(WORKLOADS[name]) == count


def test_reference_arm_json_line():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "data", "config", "impl", "cpu_baseline",
                "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 3
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"] == "tiny"


def test_exchange_and_placement_reports():
    import numpy as np

    import bench
    import combine_grouped_gemm_router_b200 as m
    from oracle import exchange_plan as xp
    rng = np.random.default_rng(5)
    D = rng.integers(0, 500, (8, 8)) * (np.arange(8) + 1)
    rep = bench.exchange_report(m, D, row_bytes=8192)
    assert rep["makespan_rows"] == xp.exchange_bound(D)
    assert rep["rotation_rows"] >= rep["makespan_rows"]
    assert rep["makespan_us_at_peer_copy"] == pytest.approx(
        rep["makespan_rows"] * 8192 / (bench.PEER_COPY_GBS * 1e3))
    counts = rng.integers(0, 9, (3, 16, 16))
    rep = bench.placement_report(m, counts, 4, 16, 4)
    assert rep["hops"] == int(counts.sum())
    assert 0.0 <= rep["cross_fraction_placed"] <= rep["cross_fraction_contiguous"] <= 1.0


def test_affine_router_leans_on_the_previous_layer():
    """Layer l's router row e is rho times the previous layer's row pi_l[e] plus independent
    noise: the correlation of matched rows is rho, and every entry keeps variance 1/d."""
    import math

    import torch

    from moe_workloads import WORKLOADS, affine_router, make_layer_inputs
    w = WORKLOADS["stack4_affinity"].with_(N=64, d=1024, f=128)
    r0, r1 = affine_router(w, 0, 0), affine_router(w, 0, 1)
    assert float(r1.var()) * w.d == pytest.approx(1.0, rel=0.05)
    corr = (r1 @ r0.T) / (r1.norm(dim=1, keepdim=True) * r0.norm(dim=1)[None, :])
    best = corr.max(dim=1).values
    assert float(best.mean()) == pytest.approx(w.affinity, abs=0.02)
    assert sorted(corr.argmax(dim=1).tolist()) == list(range(w.E))   # a permutation
    # the expert weights are the plain stack's: the draw order is unchanged
    plain = make_layer_inputs(w.with_(affinity=0.0), seed=0, layer=1, with_x=False)
    planted = make_layer_inputs(w, seed=0, layer=1, with_x=False)
    assert torch.equal(plain["w2"], planted["w2"])
    assert torch.equal(planted["w_router"], r1)
    assert not math.isclose(float((plain["w_router"] - r1).abs().max()), 0.0)


def test_traffic_gate_ignores_comments_only(tmp_path):
    """The bench reports measured DRAM traffic only for the kernel code it was measured on:
    an edit to comments or whitespace keeps the figure, an edit to code drops it."""
    import bench
    src = tmp_path / "k.cuh"
    src.write_text("// header\nint f(int a) { return a + 1; }  /* note */\n")
    h0 = bench.kernel_source_hash(str(src))
    src.write_text("// header, reworded\n\nint f(int a)   { return a + 1; }\n")
    assert bench.kernel_source_hash(str(src)) == h0
    src.write_text("// header\nint f(int a) { return a + 2; }\n")
    assert bench.kernel_source_hash(str(src)) != h0
    # a figure is reported only while the kernel source hashes to the captured one
    for name, (sha, nbytes) in bench.MEASURED_UP_TRAFFIC.items():
        cur = bench.kernel_source_hash(os.path.join(bench.ROOT, "combine_grouped_gemm_router_b200",
                                                    "csrc", "grouped_gemm.cuh"))
        assert bench.up_traffic(name) == (nbytes if sha == cur else None)


def test_algorithmic_work_counts_the_payload_and_output_bytes():
    """The combine's algorithmic bytes follow what it reads and writes: fp32 expert rows or the
    FP8 return payload (d codes + d/32 exponent bytes per row), and the bf16 layer output."""
    import bench
    from moe_workloads import WORKLOADS
    w = WORKLOADS["e128_skew_fp8"]
    R, N, d, K = 21185, w.N, w.d, w.K
    plain = bench.algorithmic_work(w, R, 128)["combine_bytes"]
    ret = bench.algorithmic_work(w.with_(fp8_return=True), R, 128)["combine_bytes"]
    assert plain == R * d * 4 + N * K * 8 + N * d * 2
    assert ret == R * (d + d // 32) + N * K * 8 + N * d * 2
    up = bench.algorithmic_work(WORKLOADS["mixtral_prefill"], 8192, 8)
    assert up["up_flops"] == 4.0 * 4096 * 14336 * 8192
    assert up["up_bytes"] == 2.0 * 8 * 14336 * 4096 * 2 + 8192 * 4096 * 2 + 8192 * 14336 * 2


def test_workload_selection_and_payload_bytes():
    """The bench runs the bf16-path workloads with the fp16 return payload unless --y-f32, keeps
    the FP8 workloads' own payloads, and counts the combine's payload bytes accordingly
    (2d code bytes + d/32 exponent bytes per kept row)."""
    import bench
    w = bench.select_workload(bench.parse([]))
    assert w.name == "stack4" and w.y_f16 and not w.fp8
    assert not bench.select_workload(bench.parse(["--y-f32"])).y_f16
    assert not bench.select_workload(bench.parse(["--workload", "e128_skew_fp8"])).y_f16
    assert bench.select_workload(bench.parse(["--workload", "decode", "--tokens", "8"])).N == 8
    w = bench.select_workload(bench.parse(["--workload", "e128_skew"]))
    R, N, d, K = 21185, w.N, w.d, w.K
    assert bench.algorithmic_work(w, R, 128)["combine_bytes"] == \
        R * (2 * d + d // 32) + N * K * 8 + N * d * 2
