"""Multi-rank plumbing of the benchmark on CPU (gloo).

Streams are independent (section 4.1 of the paper: no data dependencies
across (b, r) pairs), so a job's streams are split into contiguous ranges,
one per rank, and nothing is exchanged on the data path.  These tests check
the split itself (every stream owned by exactly one rank, whole batch
elements where the workload has value rows), that the ranks' per-slice
results concatenate to the one-rank result, and the timing reductions (the
slowest rank's time, the units all ranks processed).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_world(target, world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q) + args) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res, key=lambda r: r[0])


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))


def _reduce_worker(rank, world, port, q):
    _init(rank, world, port)
    import bench
    ms, units = bench.reduce_over_ranks(10.0 + 5.0 * rank, 1000.0 * (rank + 1))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms, units))


def test_reduce_over_ranks_gloo_world2():
    for rank, ms, units in _run_world(_reduce_worker, 2):
        assert ms == 15.0          # max over ranks
        assert units == 3000.0     # sum over ranks


def test_reduce_single_process_is_identity():
    import bench
    assert bench.reduce_over_ranks(3.5, 42.0) == (3.5, 42.0)


@pytest.mark.parametrize("units,world", [(128, 1), (128, 2), (128, 8), (8, 3), (1, 2), (2048, 8), (64, 7)])
def test_shard_range_covers_every_unit_once(units, world):
    import bench
    seen = []
    sizes = []
    for r in range(world):
        lo, hi = bench.shard_range(units, world, r)
        assert 0 <= lo <= hi <= units
        seen.extend(range(lo, hi))
        sizes.append(hi - lo)
    assert seen == list(range(units))               # contiguous, in rank order, each once
    assert max(sizes) - min(sizes) <= 1             # balanced


def test_shard_plan_respects_batches_with_value_rows():
    import bench
    # markov-4-train: B = 8 batch elements of R = 256 routes, value rows -> whole batch elements
    owned = []
    for r in range(4):
        kind, lo, hi = bench.shard_plan(8, 256, True, 4, r)
        assert kind == "batches"
        owned.extend(range(lo * 256, hi * 256))
    assert owned == list(range(8 * 256))
    # qwen-proj-64: one batch element with value rows -> ranges of routes
    assert bench.shard_plan(1, 64, True, 2, 1) == ("routes", 32, 64)
    # planted-16: no value rows -> plain stream ranges across batch elements
    assert bench.shard_plan(4, 32, False, 3, 0) == ("streams", 0, 43)


def _slice_worker(rank, world, port, q, qs, ks, g):
    """Each rank runs the oracle on its contiguous slice; rank 0 assembles."""
    _init(rank, world, port)
    import bench
    import oracle
    lo, hi = bench.shard_range(qs.shape[0], world, rank)
    part = oracle.match_sam(qs[lo:hi], ks[lo:hi], g=g, threads=1)
    parts = [None] * world
    dist.all_gather_object(parts, (lo, hi, [p.tolist() for p in part]))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, parts))


def test_stream_slices_concatenate_to_the_one_rank_result():
    from suffix_automaton_retrieval_b200 import workloads as W
    import oracle
    oracle.build()
    w = W.zipf_planted(S=10, T=3000, lmax=200)
    whole = oracle.match_sam(w.q, w.k, g=w.g, threads=1)
    res = _run_world(_slice_worker, 2, w.q, w.k, w.g)
    parts = res[0][1]
    assert [p[:2] for p in parts] == [(0, 5), (5, 10)]
    for i, name in enumerate(("end_idx", "len", "sym")):
        got = np.concatenate([np.asarray(p[2][i], np.int32) for p in parts])
        assert np.array_equal(got, whole[i]), name
