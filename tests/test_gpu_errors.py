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
                m.w2_for(shape, inp["w2"].cuda()), out, stats=stats, ws=ws)
    assert m.moe_get_device_error(True) == 7  # MOE_ERR_NONFINITE
    assert m.read_stats(stats).nonfinite_tokens == 1


def test_empty_batch_every_entry_point():
    """N = 0 (an empty batch) is a valid call: every entry point returns OK, launches nothing,
    and the outputs indexed by expert or rank come back zero."""
    import combine_grouped_gemm_router_b200 as m
    dev = torch.device("cuda")
    E, K, W, d, f = 8, 2, 4, 128, 256
    for flags in ({}, {"slot_major": True}, {"reroute": True, "capacity_factor": 1.0}):
        shape = m.make_shape(0, d, f, E, K, W, **flags)
        ws = torch.empty(max(m.moe_layer_workspace_size(shape), 256), dtype=torch.uint8,
                         device=dev)
        empty = lambda *sz, dt=torch.float32: torch.empty(*sz, dtype=dt, device=dev)
        x = empty(0, d, dt=torch.bfloat16)
        topk = empty(0, K, dt=torch.int32)
        tw = empty(0, K)
        logits = empty(0, E)
        m.moe_route(shape, x, torch.randn(E, d, device=dev), None, topk, tw, logits, ws)
        counts = torch.full((E,), 7, dtype=torch.int32, device=dev)
        kept = torch.full((E,), 7, dtype=torch.int32, device=dev)
        offsets = torch.full((E + 1,), 7, dtype=torch.int32, device=dev)
        D = torch.full((W * W,), 7, dtype=torch.int64, device=dev)
        pk = torch.full((W * W + 1,), 7, dtype=torch.int64, device=dev)
        stats = torch.full_like(m.stats_buffer(dev), 7)
        RA = m.moe_rows_alloc(shape)
        xs = empty(RA, d, dt=torch.bfloat16)
        row_of = empty(0, dt=torch.int32)
        assign = empty(RA, dt=torch.int32)
        if flags.get("reroute"):
            m.moe_dispatch_reroute(shape, x, logits, topk, counts, kept, offsets, row_of, assign, xs,
                                   rank_matrix=D, packed_offsets=pk, stats=stats, ws=ws)
        else:
            m.moe_dispatch(shape, x, topk, counts, kept, offsets, row_of, assign, xs, None, D, pk,
                           stats, ws)
        torch.cuda.synchronize()
        for t in (counts, kept, offsets, D, pk, stats):
            assert int(t.abs().sum().item()) == 0
        w1 = torch.zeros(E, f, d, dtype=torch.bfloat16, device=dev)
        w2 = torch.zeros(E, d, f, dtype=torch.bfloat16, device=dev)
        h = empty(RA, f, dt=torch.bfloat16)
        y = empty(RA, d)
        m.moe_expert_gemm(shape, xs, offsets, w1, w1, w2, h, y)
        out = empty(0, d)
        m.moe_combine(shape, y, row_of, tw, out)
        stats2 = torch.full_like(m.stats_buffer(dev), 7)
        m.moe_layer(shape, x, torch.randn(E, d, device=dev), None, w1, w1, w2, out, stats=stats2,
                    ws=ws)
        torch.cuda.synchronize()
        assert int(stats2.abs().sum().item()) == 0
        m.moe_affinity_accumulate(0, E, K, topk, topk, torch.zeros(E, E, dtype=torch.int64,
                                                                  device=dev))
    assert m.moe_get_device_error(True) == 0
