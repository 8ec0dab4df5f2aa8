"""The layer over W real ranks (combine_grouped_gemm_router_b200.ranks.layer_ranks), run as 2-4
gloo ranks on the CPU. The orchestration is the library's (route, all-gather of the top-K, the
dispatch of each rank, the all-to-allv of the packed rows, the regroup, the experts, the way
back, the return all-to-allv, the combine); the kernels are stood in for by the oracle under the
same contracts (the GPU test tests/test_gpu_ranks.py holds the kernels to those contracts). Every
rank's routing, traffic matrix and bookkeeping must equal the oracle's one-process layer of the
whole batch, bit for bit, and every token's output must equal it up to fp64 rounding."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The kernels' contracts on CPU tensors, by the oracle (test infrastructure)."""

    def __init__(self):
        import oracle
        from combine_grouped_gemm_router_b200 import MoeShape
        oracle.build()
        self.orc = oracle
        self.MoeShape = MoeShape

    def route(self, local, x, w_router, bias):
        import torch
        lg = self.orc.router_logits(x, w_router, bias)
        idx, w, _ = self.orc.topk(lg, local.K)
        return torch.from_numpy(idx), torch.from_numpy(w)

    def dispatch_rank(self, shape, rank, x_local, topk_all):
        import torch
        N, E, K, W, d = shape.N, shape.E, shape.K, shape.W, shape.d
        S = N // W
        C = min(self.orc.capacity(N, E, K, shape.capacity_factor), N * K)
        p = self.orc.positions(topk_all.numpy(), E, W, C, order=int(bool(shape.flags & 2)))
        pk_off, pr = p["pk_off"], p["packed_row_of"]
        base = int(pk_off[rank * W])
        n_send = int(pk_off[(rank + 1) * W]) - base
        x_send = torch.zeros(n_send + 128, d, dtype=torch.bfloat16)
        local = pr[rank * S * K:(rank + 1) * S * K]
        for i in np.nonzero(local >= 0)[0]:
            x_send[int(local[i]) - base] = x_local[i // K]
        return dict(counts=p["counts"], kept=p["kept"], offsets=p["offsets"], row_of=p["row_of"],
                    assign=p["assign_of_row"], packed_row_of=pr,
                    send_row_of=torch.from_numpy(np.where(local >= 0, local - base, -1)),
                    x_send=x_send, D=torch.from_numpy(p["D"].reshape(-1).copy()),
                    pk_off=pk_off)

    def regroup(self, shape, rank, direction, src, book, rows):
        """The contract of moe_regroup_rows."""
        W, E, K = shape.W, shape.E, shape.K
        S, El = shape.N // W, E // W
        D = book["D"].numpy().reshape(W, W)
        pk_off = book["pk_off"]
        base = [int(D[:i, rank].sum()) - int(pk_off[i * W + rank]) for i in range(W)]
        offs = book["offsets"]
        lo, hi = int(offs[rank * El]), int(offs[(rank + 1) * El])
        dst = src.new_zeros((rows + (128 if direction == 0 else 0),) + tuple(src.shape[1:]))
        for r in range(lo, hi):
            a = int(book["assign"][r])
            recv = base[(a // K) // S] + int(book["packed_row_of"][a])
            if direction == 0:
                dst[r - lo] = src[recv]
            else:
                dst[recv] = src[r - lo]
        import torch
        return dst, torch.from_numpy((offs[rank * El:(rank + 1) * El + 1] - lo).astype(np.int32))

    def experts(self, shape, rank, x_sorted, offsets_local, rows, w1, w3, w2):
        import torch
        off = offsets_local.numpy()
        row_expert = np.repeat(np.arange(len(off) - 1, dtype=np.int32), np.diff(off))
        _, y = self.orc.expert_rows(np.arange(rows, dtype=np.int32), row_expert, x_sorted[:rows],
                                    w1, w3, w2)
        out = torch.zeros(rows + 128, shape.d, dtype=torch.float64)
        out[:rows] = torch.from_numpy(y)
        return out

    def combine(self, local, y, row_of, topk_w, residual, out):
        import torch
        ro = row_of.numpy()
        y_of_slot = np.zeros((ro.size, local.d))
        y_of_slot[ro >= 0] = y.numpy()[ro[ro >= 0]]
        out.copy_(torch.from_numpy(self.orc.combine(ro, topk_w.numpy(), y_of_slot)))
        return out


def _worker(rank, world, port, wl, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    import combine_grouped_gemm_router_b200 as m
    from combine_grouped_gemm_router_b200.ranks import layer_ranks
    from moe_workloads import make_layer_inputs
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    try:
        inp = make_layer_inputs(wl, seed=3)  # every rank draws the same inputs, keeps its share
        S, El = wl.N // world, wl.E // world
        shape = m.make_shape(wl.N, wl.d, wl.f, wl.E, wl.K, world, wl.cf, slot_major=wl.slot_major)
        out = torch.empty(S, wl.d, dtype=torch.float64)
        sl = slice(rank * El, (rank + 1) * El)
        book = layer_ranks(shape, inp["x"][rank * S:(rank + 1) * S], inp["w_router"], inp["bias"],
                           inp["w1"][sl], inp["w3"][sl], inp["w2"][sl], out, ops=OracleOps())
        q.put((rank, out.numpy(), book["topk_all"].numpy(), book["D_host"].numpy(),
               np.asarray(book["row_of"]), np.asarray(book["send_row_of"]), None))
    except Exception as e:  # report, do not hang the other ranks' queue reads
        import traceback
        q.put((rank, None, None, None, None, None, traceback.format_exc()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,wl", [
    (2, ("two", 64, 128, 128, 8, 2, 0.0, 0.0, False)),
    (4, ("four_drop", 96, 128, 128, 8, 3, 1.0, 1.1, False)),
    (3, ("three_slot", 60, 128, 128, 6, 2, 0.75, 0.5, True)),
], ids=["2-dropless", "4-drops", "3-slot-major"])
def test_layer_ranks_matches_one_process_layer(orc, world, wl):
    from moe_workloads import Workload, make_layer_inputs
    name, N, d, f, E, K, cf, s, slot = wl
    w = Workload(name, N=N, d=d, f=f, E=E, K=K, W=world, cf=cf, s=s, slot_major=slot)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, w, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted((q.get(timeout=300) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in results:
        assert r[-1] is None, r[-1]
    ref = orc.layer(make_layer_inputs(w, seed=3), K, world, cf, order=int(slot))
    out = np.concatenate([r[1] for r in results], 0)
    S = N // world
    for rank, _, topk_all, D, row_of, send_row_of, _ in results:
        np.testing.assert_array_equal(topk_all, ref["topk_idx"])
        np.testing.assert_array_equal(D, ref["D"])
        np.testing.assert_array_equal(row_of, ref["row_of"])
        pr = ref["packed_row_of"][rank * S * K:(rank + 1) * S * K]
        base = ref["pk_off"][rank * world]
        np.testing.assert_array_equal(send_row_of, np.where(pr >= 0, pr - base, -1))
    np.testing.assert_allclose(out, ref["out"], rtol=1e-12, atol=1e-12)
