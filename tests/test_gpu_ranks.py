"""The layer over W real ranks (moe_dispatch_rank, moe_regroup_rows), on one GPU: the ranks run
one after another (no kernel waits for another rank) and the two exchanges are done by the test
as row copies between the ranks' buffers, in the order the all-to-allv delivers them (blocks by
source rank, each in its sender's order). Checked against the one-GPU layer of the whole batch:
the bookkeeping bit for bit on every rank, each rank's send rows equal to the one-GPU packed
buffer's block row, each rank's regrouped rows equal to the one-GPU expert-sorted rows of its
experts, its expert outputs equal to the one-GPU y rows, and the layer output of every token
within the stated tolerance of the one-GPU layer's (and of the oracle's)."""
import numpy as np
import pytest
import torch

from layer_runner import assert_within_tolerance, lib, run_stages
from moe_workloads import Workload, make_layer_inputs

pytestmark = pytest.mark.gpu

CASES = [
    Workload("ranks2", N=256, d=256, f=256, E=8, K=2, W=2),
    Workload("ranks4_drop", N=512, d=256, f=128, E=16, K=3, W=4, cf=1.0, s=1.1),
    Workload("ranks8_slot", N=1024, d=128, f=256, E=32, K=4, W=8, cf=1.25, s=0.8,
             slot_major=True),
    Workload("ranks8_pairs", N=4096, d=512, f=256, E=8, K=2, W=8),  # >= 768 rows per expert
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_ranks_layer_matches_one_gpu_layer(orc, w):
    m = lib()
    dev = torch.device("cuda")
    inp = make_layer_inputs(w, seed=0)
    one = run_stages(inp, w)                    # the whole batch on one GPU (W virtual ranks)
    assert one["dev_error"] == 0
    shape = m.make_shape(w.N, w.d, w.f, w.E, w.K, w.W, w.cf, slot_major=w.slot_major)
    N, K, E, W, d = w.N, w.K, w.E, w.W, w.d
    S, El = N // W, E // W
    x = inp["x"].to(dev)
    bias = None if inp["bias"] is None else inp["bias"].to(dev)
    from combine_grouped_gemm_router_b200.ranks import CudaOps
    ops = CudaOps()
    local = m.MoeShape(S, d, w.f, E, K, 1, w.cf, shape.flags)
    # 1. every rank routes its own tokens; the top-K is gathered
    routes = [ops.route(local, x[r * S:(r + 1) * S], inp["w_router"].to(dev), bias)
              for r in range(W)]
    topk_all = torch.cat([t for t, _ in routes], 0)
    assert torch.equal(topk_all, one["topk_idx"])
    # 2. every rank's dispatch: the whole batch's bookkeeping, its own send rows
    books = [ops.dispatch_rank(shape, r, x[r * S:(r + 1) * S], topk_all) for r in range(W)]
    torch.cuda.synchronize()
    assert m.moe_get_device_error(True) == 0
    R = int(one["offsets"][E].item())
    pk_off = one["pk_off"].cpu().numpy()
    Dh = one["D"].cpu().numpy().reshape(W, W)
    for r, b in enumerate(books):
        for key in ("counts", "kept", "offsets", "row_of"):
            assert torch.equal(b[key], one[key]), (r, key)
        assert torch.equal(b["assign"][:R], one["assign"][:R]), r
        assert torch.equal(b["D"], one["D"]) and torch.equal(b["pk_off"], one["pk_off"]), r
        n_send = int(Dh[r].sum())
        assert torch.equal(b["x_send"][:n_send], one["x_packed"][pk_off[r * W]:pk_off[r * W] + n_send])
        # send_row_of: each local slot's row in the send buffer
        sro = b["send_row_of"].cpu().numpy()
        pro = b["packed_row_of"].cpu().numpy()[r * S * K:(r + 1) * S * K]
        np.testing.assert_array_equal(sro, np.where(pro >= 0, pro - pk_off[r * W], -1))
    # 3. the exchange: rank j receives block (i, j) of every i, in order of i
    recv = []
    for j in range(W):
        parts = []
        for i in range(W):
            a0 = int(Dh[i, :j].sum())
            parts.append(books[i]["x_send"][a0:a0 + int(Dh[i, j])])
        recv.append(torch.cat(parts, 0))
    # 4. regroup into each rank's experts' order, the experts, the way back
    offs = one["offsets"].cpu().numpy()
    w1, w3 = inp["w1"].to(dev), inp["w3"].to(dev)
    w2 = m.w2_for(shape, inp["w2"].to(dev))
    y_back = []
    for j in range(W):
        rows = recv[j].shape[0]
        xs, off_l = ops.regroup(shape, j, 0, recv[j], books[j], rows)
        lo, hi = int(offs[j * El]), int(offs[(j + 1) * El])
        assert rows == hi - lo
        assert torch.equal(xs[:rows], one["x_sorted"][lo:hi]), j
        np.testing.assert_array_equal(off_l.cpu().numpy(), offs[j * El:(j + 1) * El + 1] - lo)
        y = ops.experts(shape, j, xs, off_l, rows, w1[j * El:(j + 1) * El],
                        w3[j * El:(j + 1) * El], w2[j * El:(j + 1) * El])
        yb, _ = ops.regroup(shape, j, 1, y[:rows], books[j], rows)
        torch.cuda.synchronize()
        # the same rows, the same weights: the one-GPU expert outputs (within fp32 accumulation)
        assert_within_tolerance(y[:rows], one["y"][lo:hi], f"y of rank {j}")
        y_back.append(yb)
    # 5. the return exchange: rank i receives block (i, j) of every j, in order of j
    outs = []
    for i in range(W):
        parts = []
        for j in range(W):
            a0 = int(Dh[:i, j].sum())
            parts.append(y_back[j][a0:a0 + int(Dh[i, j])])
        y_ret = torch.cat(parts, 0)
        out = torch.empty(S, d, dtype=torch.float32, device=dev)
        ops.combine(local, y_ret, books[i]["send_row_of"], routes[i][1], None, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(True) == 0
    out = torch.cat(outs, 0)
    assert_within_tolerance(out, one["out"], "W-rank layer vs one-GPU layer")
    ref = orc.layer(inp, K, W, w.cf, order=int(w.slot_major))
    rep = assert_within_tolerance(out, ref["out"], "W-rank layer vs oracle")
    print(w.name, rep, "bitwise equal to one GPU:", bool(torch.equal(out, one["out"])))
