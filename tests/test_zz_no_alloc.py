"""moe_dispatch_static: the dispatch entry point for callers that cannot allocate device
memory (a plugin whose host owns every allocation, a process with a device-memory budget fixed
at start-up, a latency-critical loop that cannot afford a cudaMalloc). It uses a fixed
scratch array inside the library instead of a caller workspace.

Checked here through the C ABI: on two calls in a row, its outputs equal those of the
workspace-taking moe_dispatch bit for bit (integer bookkeeping and row copies, the same
tolerance every dispatch test uses), and a shape whose scratch does not fit the array is
rejected before anything runs. This file is collected last and also runs on its own."""
import pytest
import torch

from moe_workloads import WORKLOADS, Workload, zipf_bias

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    from combine_grouped_gemm_router_b200 import build
    build.build()
    import combine_grouped_gemm_router_b200 as mod
    mod.moe_get_device_error(True)
    return mod


def _buffers(m, shape, w, dev):
    RA = m.moe_rows_alloc(shape)
    return dict(
        counts=torch.full((w.E,), -1, dtype=torch.int32, device=dev),
        kept=torch.full((w.E,), -1, dtype=torch.int32, device=dev),
        offsets=torch.full((w.E + 1,), -1, dtype=torch.int32, device=dev),
        row_of=torch.full((w.N * w.K,), -9, dtype=torch.int32, device=dev),
        assign=torch.full((RA,), -9, dtype=torch.int32, device=dev),
        x_sorted=torch.zeros(RA, w.d, dtype=torch.bfloat16, device=dev),
        x_packed=torch.zeros(RA, w.d, dtype=torch.bfloat16, device=dev),
        D=torch.full((w.W * w.W,), -1, dtype=torch.int64, device=dev),
        pk_off=torch.full((w.W * w.W + 1,), -1, dtype=torch.int64, device=dev),
        stats=m.stats_buffer(dev),
    )


def _same(a: dict, b: dict, R: int):
    for k in ("counts", "kept", "offsets", "row_of", "D", "pk_off"):
        assert torch.equal(a[k], b[k]), k
    assert torch.equal(a["assign"][:R], b["assign"][:R])
    assert torch.equal(a["x_sorted"][:R], b["x_sorted"][:R])
    assert torch.equal(a["x_packed"][:R], b["x_packed"][:R])
    assert torch.equal(a["stats"], b["stats"])


@pytest.mark.parametrize("w", [
    WORKLOADS["tiny"],
    Workload("ragged_drop", N=1040, d=256, f=128, E=8, K=2, W=4, cf=0.75, s=1.1),
    WORKLOADS["e128_skew"],
    WORKLOADS["stack4"].with_(cf=1.0, s=1.2),
], ids=lambda w: w.name)
def test_static_scratch_dispatch_matches_workspace_dispatch(m, w):
    dev = torch.device("cuda")
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf)
    g = torch.Generator(device=dev).manual_seed(7)
    x = torch.randn(w.N, w.d, generator=g, device=dev).to(torch.bfloat16)
    wr = torch.randn(w.E, w.d, generator=g, device=dev) / w.d ** 0.5
    bias = zipf_bias(w.E, w.s)
    bias = None if bias is None else bias.to(dev)
    topk = torch.empty(w.N, w.K, dtype=torch.int32, device=dev)
    topw = torch.empty(w.N, w.K, dtype=torch.float32, device=dev)
    ws = torch.empty(m.moe_workspace_size(shape), dtype=torch.uint8, device=dev)
    m.moe_route(shape, x, wr, bias, topk, topw, None, ws)

    ref = _buffers(m, shape, w, dev)
    m.moe_dispatch(shape, x, topk, ref["counts"], ref["kept"], ref["offsets"], ref["row_of"],
                   ref["assign"], ref["x_sorted"], ref["x_packed"], ref["D"], ref["pk_off"],
                   ref["stats"], ws)
    torch.cuda.synchronize()
    R = int(ref["offsets"][w.E].item())
    for call in range(2):  # two calls in a row share the library's scratch array
        got = _buffers(m, shape, w, dev)
        m.moe_dispatch_static(shape, x, topk, got["counts"], got["kept"], got["offsets"],
                              got["row_of"], got["assign"], got["x_sorted"], got["x_packed"],
                              got["D"], got["pk_off"], got["stats"])
        torch.cuda.synchronize()
        _same(ref, got, R)
    # with the traffic matrix and pack offsets left to the scratch array as well: every other
    # output still bit for bit (a wrong pack-offset layout inside the array would show in
    # x_packed, a wrong counter write in stats)
    got = _buffers(m, shape, w, dev)
    m.moe_dispatch_static(shape, x, topk, got["counts"], got["kept"], got["offsets"],
                          got["row_of"], got["assign"], got["x_sorted"], got["x_packed"],
                          stats=got["stats"])
    torch.cuda.synchronize()
    for k in ("counts", "kept", "offsets", "row_of", "stats"):
        assert torch.equal(ref[k], got[k]), k
    for k in ("assign", "x_sorted", "x_packed"):
        assert torch.equal(ref[k][:R], got[k][:R]), k
    assert m.moe_get_device_error(True) == 0


def test_static_scratch_rejects_oversized_shapes(m):
    # E * blocks * 4 bytes of histograms alone exceeds the 1 MiB array
    big = m.make_shape(1 << 20, 128, 128, 256, 1, 1, 0.0)
    P = 0x100000  # never dereferenced: the size check comes first
    import ctypes
    rc = m._lib.moe_dispatch_static(ctypes.byref(big), P, P, P, P, P, P, P, P, None, None, None,
                                    None, None)
    assert rc == 3  # MOE_ERR_WORKSPACE_TOO_SMALL
    with pytest.raises(m.MoeError):
        m.moe_dispatch_static(big, P, P, P, P, P, P, P, P)
