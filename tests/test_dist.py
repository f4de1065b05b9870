"""Multi-rank plumbing of the benchmark on CPU (gloo, world size 2).

Streams are independent, so ranks exchange nothing on the data path; the
only collectives are the timing reductions: the slowest rank's time and the
units all ranks processed.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    ms, units = bench.reduce_over_ranks(10.0 + 5.0 * rank, 1000.0 * (rank + 1))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms, units))


def test_reduce_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, units in res:
        assert ms == 15.0          # max over ranks
        assert units == 3000.0     # sum over ranks


def test_reduce_single_process_is_identity():
    import bench
    assert bench.reduce_over_ranks(3.5, 42.0) == (3.5, 42.0)
