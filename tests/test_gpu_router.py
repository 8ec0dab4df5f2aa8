"""Parity of the router with the oracle, through moe_route: the fused kernels (projection + top-K
in one kernel: many tokens, E >= 32; the broadcast form for E = 32 and the split-warp form on
the transposed weights for E > 32, in each of its tile configurations: 64 experts with 2 or 4
tokens per lane, 128 and 256 experts) and the separate kernels (few logits: small N or few
experts, then the top-K kernel). Checked: the logits bit for bit (each one fp32 fmaf chain over d
in ascending order from +0, then + bias), the top-K indices exactly, the gate weights within fp32
rounding of the oracle's fp64 softmax. The shapes cover a ragged last token tile, hidden sizes
that are not a multiple of the staged chunk (32 or 64 elements), every padded expert width (E
rounded up to 32, 64, 128, 256), K from 1 to 32, with and without a bias, and planted ties (two
experts with identical router rows: equal logits, the lower expert index first)."""
import numpy as np
import pytest
import torch

from moe_workloads import Workload, make_layer_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # (N, d, E, K, zipf s)
    (2048, 128, 32, 1, 0.0),
    (2050, 200, 48, 6, 1.1),     # ragged last tile; d = 6 chunks of 32 + 8
    (2080, 256, 64, 6, 0.0),
    (2111, 136, 100, 8, 0.7),    # E padded to 128
    (4096, 512, 128, 8, 1.1),
    (2048, 1024, 160, 32, 0.0),  # E padded to 256, K = 32
    (2049, 64, 256, 8, 1.2),
    (2080, 328, 200, 8, 0.0),    # E padded to 256, d = 5 chunks of 64 + 8
    (2048, 8, 128, 4, 0.0),      # a single ragged chunk
    # the split-warp form with 4 tokens per lane (E <= 64, several CTAs per SM): ragged last
    # tile, partial chunk, padded experts
    (30000, 136, 64, 6, 1.2),
    (29001, 256, 40, 4, 0.0),
    # the separate kernels: decode-sized, few experts, an odd expert count, one token
    (16, 7168, 256, 8, 0.0),
    (4096, 512, 8, 2, 0.0),
    (100, 136, 5, 2, 0.9),
    (33, 64, 20, 3, 0.0),
    (1, 8, 1, 1, 0.0),
]


def _route(m, shape, x, wr, bias):
    dev = x.device
    N, K, E = shape.N, shape.K, shape.E
    topk = torch.empty(N, K, dtype=torch.int32, device=dev)
    topw = torch.empty(N, K, dtype=torch.float32, device=dev)
    logits = torch.empty(N, E, dtype=torch.float32, device=dev)
    ws = torch.empty(max(m.moe_workspace_size(shape), 256), dtype=torch.uint8, device=dev)
    m.moe_route(shape, x, wr, bias, topk, topw, logits, ws)
    torch.cuda.synchronize()
    return topk.cpu().numpy(), topw.cpu().numpy(), logits.cpu().numpy()


@pytest.mark.parametrize("case", CASES, ids=lambda c: "N%d_d%d_E%d_K%d" % c[:4])
def test_router_matches_oracle(orc, case):
    import combine_grouped_gemm_router_b200 as m
    N, d, E, K, s = case
    w = Workload("router", N=N, d=d, f=8, E=E, K=K, W=1, s=s)
    inp = make_layer_inputs(w, seed=5)
    wr = inp["w_router"].clone()
    tie = E > 4
    if tie:
        wr[E - 1] = wr[3]  # planted tie: experts 3 and E-1 always have equal logits
    dev = torch.device("cuda")
    shape = m.make_shape(N, d, 8, E, K, 1)
    bias = inp["bias"]
    if bias is not None and tie:
        bias = bias.clone()
        bias[E - 1] = bias[3]
    topk, topw, logits = _route(m, shape, inp["x"].to(dev), wr.to(dev),
                                None if bias is None else bias.to(dev))
    assert m.moe_get_device_error(True) == 0
    ref_logits = orc.router_logits(inp["x"], wr, bias)
    assert np.array_equal(logits.view(np.uint32), ref_logits.view(np.uint32)), \
        "logits differ in %d places" % int((logits != ref_logits).sum())
    ref_idx, ref_w, nonfinite = orc.topk(ref_logits, K)
    assert nonfinite == 0
    np.testing.assert_array_equal(topk, ref_idx)
    np.testing.assert_allclose(topw, ref_w, rtol=2e-6, atol=1e-7)
    # the tie: wherever both tied experts are chosen, the lower index comes first
    both = (topk == 3).any(1) & (topk == E - 1).any(1) & tie
    for t in np.nonzero(both)[0]:
        row = list(topk[t])
        assert row.index(3) < row.index(E - 1)


def test_fused_router_flags_nonfinite_tokens(orc):
    """A token whose hidden state holds an infinity gets non-finite logits: the sticky error
    word records it, the other tokens' results are unaffected."""
    import combine_grouped_gemm_router_b200 as m
    N, d, E, K = 2048, 128, 64, 4
    w = Workload("router_inf", N=N, d=d, f=8, E=E, K=K, W=1)
    inp = make_layer_inputs(w, seed=6)
    x = inp["x"].clone()
    x[77, 5] = float("inf")
    dev = torch.device("cuda")
    shape = m.make_shape(N, d, 8, E, K, 1)
    m.moe_get_device_error(True)
    topk, topw, logits = _route(m, shape, x.to(dev), inp["w_router"].to(dev), None)
    assert m.moe_get_device_error(True) == 7  # MOE_ERR_NONFINITE
    ref_logits = orc.router_logits(x, inp["w_router"], None)
    keep = np.ones(N, bool)
    keep[77] = False
    assert np.array_equal(logits[keep].view(np.uint32), ref_logits[keep].view(np.uint32))
    ref_idx, _, _ = orc.topk(ref_logits[keep], K)
    np.testing.assert_array_equal(topk[keep], ref_idx)
