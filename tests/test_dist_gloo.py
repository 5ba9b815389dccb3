"""Multi-rank host logic of bench.py on CPU: two gloo ranks aggregate their
step times (max) and work (sum) exactly as the GPU ranks do over NCCL."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms, flops = bench.aggregate(10.0 + rank, 1e12 * (rank + 1), world)
    q.put((rank, ms, flops))
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, flops in out:
        assert ms == 11.0            # max over ranks
        assert flops == 3e12         # sum over ranks


def test_aggregate_single_rank_is_identity():
    import bench
    assert bench.aggregate(5.0, 7.0, 1) == (5.0, 7.0)
