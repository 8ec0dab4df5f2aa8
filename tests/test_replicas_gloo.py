"""The N>1 path of the bench: independent replicas per rank, the reported time is
the max over ranks and the value counts every rank's tokens. Run as two gloo
ranks on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist
    bench.init_dist("gloo")
    elapsed = [0.5, 2.0][rank]
    tokens = [4096.0, 4096.0][rank]
    agg = bench.aggregate(tokens, elapsed)
    bench.barrier()
    # the reference arm runs on rank 0 only; other ranks return without work
    args = bench.parse(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    ref = bench.run_reference(args, None) if rank != 0 else "skipped"
    q.put((rank, agg, ref))
    dist.destroy_process_group()


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, agg, ref in results:
        assert agg["elapsed_max_s"] == pytest.approx(2.0)
        assert agg["tokens_total"] == pytest.approx(8192.0)
        assert agg["value"] == pytest.approx(4096.0)
        if rank == 1:
            assert ref is None
