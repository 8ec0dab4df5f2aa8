"""Kernel-side error reporting on the GPU, with no fault: bad expert ids and
non-finite logits are recorded in the device error word; a bounded wait on a
flag nobody sets gives up and reports a timeout; the context stays usable."""
import numpy as np
import pytest
import torch

from moe_workloads import Workload, make_layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    from combine_grouped_gemm_router_b200 import build
    build.build()
    import combine_grouped_gemm_router_b200 as mod
    mod.moe_get_device_error(True)
    return mod


def test_bounded_wait_times_out_and_context_survives(m):
    m.moe_debug_bounded_wait(50_000_000)  # 50 ms
    assert m.moe_get_device_error(True) == 6  # MOE_ERR_DEVICE_TIMEOUT
    assert m.moe_get_device_error(True) == 0
    x = torch.arange(10, device="cuda").sum().item()
    assert x == 45


def test_out_of_range_expert_ids_are_flagged_not_faulted(m):
    N, E, K, W, d = 64, 8, 2, 4, 128
    shape = m.make_shape(N, d, 128, E, K, W, 0.0)
    dev = "cuda"
    topk = torch.randint(0, E, (N, K), dtype=torch.int32, device=dev)
    topk[3, 1] = E + 5
    topk[10, 0] = -2
    RA = m.moe_rows_alloc(shape)
    ws = torch.empty(m.moe_workspace_size(shape), dtype=torch.uint8, device=dev)
    x = torch.randn(N, d, device=dev).to(torch.bfloat16)
    bufs = [torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E, dtype=torch.int32, device=dev),
            torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(N * K, dtype=torch.int32, device=dev),
            torch.empty(RA, dtype=torch.int32, device=dev)]
    xs = torch.empty(RA, d, dtype=torch.bfloat16, device=dev)
    m.moe_dispatch(shape, x, topk, *bufs, xs, ws=ws)
    assert m.moe_get_device_error(True) == 8  # MOE_ERR_DEVICE_BOUNDS
    row_of = bufs[3].cpu().numpy().reshape(N, K)
    assert row_of[3, 1] == -1 and row_of[10, 0] == -1
    assert bufs[0].sum().item() == N * K - 2


def test_nonfinite_logits_are_flagged(m):
    w = Workload("nan", N=32, d=128, f=128, E=8, K=2, W=4)
    inp = make_layer_inputs(w, seed=0)
    x = inp["x"].clone()
    x[5, 7] = float("nan")
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, 0.0)
    ws = torch.empty(m.moe_layer_workspace_size(shape), dtype=torch.uint8, device="cuda")
    out = torch.empty(w.N, w.d, dtype=torch.float32, device="cuda")
    stats = m.stats_buffer()
    m.moe_layer(shape, x.cuda(), inp["w_router"].cuda(), None, inp["w1"].cuda(), inp["w3"].cuda(),
                inp["w2"].cuda(), out, stats=stats, ws=ws)
    assert m.moe_get_device_error(True) == 7  # MOE_ERR_NONFINITE
    assert m.read_stats(stats).nonfinite_tokens == 1
