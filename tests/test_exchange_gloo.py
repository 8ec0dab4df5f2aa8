"""The exchange of packed rows between ranks (combine_grouped_gemm_router_b200.exchange), run
as gloo ranks on the CPU: every rank receives exactly the rows sent to it, grouped by source in
send order, through the plain all-to-allv and through the contention-free order, and both give
the same buffer. The same code runs over NCCL on GPUs (one GPU per rank), which this suite does
not reach."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _traffic(W: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    D = rng.integers(0, 40, (W, W)) * (np.arange(W) + 1)[None, :]  # skewed receivers
    D[0, W - 1] = 0                                                 # an empty block
    return D.astype(np.int64)


def _worker(rank, world, port, seed, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    import combine_grouped_gemm_router_b200 as m
    from combine_grouped_gemm_router_b200 import exchange as ex
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        D_all = _traffic(world, seed)
        # each rank knows only its own send counts; the traffic matrix is gathered
        D = ex.gather_traffic(D_all[rank].tolist())
        assert np.array_equal(D.numpy(), D_all)
        # send rows (src, dst, index within the block, a payload value), by destination
        rows = []
        for j in range(world):
            for k in range(int(D_all[rank, j])):
                rows.append([rank, j, k, rank * 1000 + j * 100 + k])
        send = torch.tensor(rows, dtype=torch.int32).reshape(-1, 4)
        plain = ex.exchange_rows(send, D)
        ordered = ex.exchange_rows_ordered(send, D)
        sched = m.moe_exchange_schedule(D_all)
        ordered2 = ex.exchange_rows_ordered(send, D, schedule=(sched[0], sched[1]))
        q.put((rank, plain.numpy(), ordered.numpy(), ordered2.numpy(), None))
    except Exception as e:  # report, do not hang the other ranks' queue reads
        q.put((rank, None, None, None, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,seed", [(2, 0), (3, 1), (4, 2)])
def test_exchange_delivers_every_block(world, seed):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seed, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    D = _traffic(world, seed)
    for rank, plain, ordered, ordered2, err in results:
        assert err is None, err
        expect = np.array([[i, rank, k, i * 1000 + rank * 100 + k]
                           for i in range(world) for k in range(int(D[i, rank]))],
                          dtype=np.int32).reshape(-1, 4)
        np.testing.assert_array_equal(plain, expect)
        np.testing.assert_array_equal(ordered, expect)
        np.testing.assert_array_equal(ordered2, expect)


def test_ordered_exchange_rejects_a_bad_schedule_before_sending(monkeypatch):
    """A schedule that is not a matching, or does not deliver D, is refused by every rank before
    any transfer (checked here in one process as rank 0 of 2: the check needs no peers)."""
    import torch
    import torch.distributed as dist

    from combine_grouped_gemm_router_b200 import exchange as ex
    monkeypatch.setattr(dist, "get_rank", lambda group=None: 0)
    monkeypatch.setattr(dist, "get_world_size", lambda group=None: 2)
    D = torch.tensor([[0, 3], [2, 0]])
    with pytest.raises(ValueError):      # receiver 1 fed by both ranks (one to itself)
        ex.exchange_rows_ordered(torch.zeros(3, 1), D, schedule=(np.array([[1, 1]]),
                                                                 np.array([3])))
    with pytest.raises(ValueError):      # a matching, but it delivers too little
        ex.exchange_rows_ordered(torch.zeros(3, 1), D, schedule=(np.array([[1, 0]]),
                                                                 np.array([2])))
