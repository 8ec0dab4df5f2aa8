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
    ("mixtral_prefill", 11),       # pair + single-CTA launch for each GEMM
    ("mixtral_prefill_fp8", 12),   # + quantisation of h
    ("e128_skew", 9),              # ~165 rows per expert: single-CTA GEMMs only
    ("e128_skew_fp8", 10),
    ("decode", 9),
    ("e128_skew_slot_major", 10),  # 1024 blocks per expert: the per-expert scan
    ("e128_skew_reroute", 14),     # two dispatch passes and the ranking kernel
    ("stack4", 12),                # 512 blocks per expert, pair GEMMs
    ("residual_top1", 14),         # shared MLP: offsets, pair + single GEMMs twice
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
