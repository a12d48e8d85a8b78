"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on CPU.

The BATQuant path is per token, so bench.py shards it by token batch: every
rank gets its own batch against the same (replicated) weights, with no
collective on the data path. The only cross-rank steps are the barrier and the
max-over-ranks timing reduction tested here.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import workloads as wl
    try:
        # per-rank timings: rank r took (r + 1) seconds for the step, 10 * (r + 1) for e2e
        got = bench.max_over_ranks(dist, [1.0 + rank, 10.0 * (rank + 1)], "cpu")
        # the token batch differs per rank; weights and factors are shared
        inp, x = bench.rank_inputs("tiny", rank)
        base = wl.make_inputs("tiny", seed=0)
        shared = (np.array_equal(inp.A, base.A) and np.array_equal(inp.B, base.B)
                  and np.array_equal(inp.W, base.W) and np.array_equal(inp.g_lo, base.g_lo))
        dist.barrier()
        out[rank] = (got, int(x.astype(np.int64).sum()), shared)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_batches():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        assert res[r][0] == [2.0, 20.0]  # every rank sees the slowest rank's times
    assert res[0][1] != res[1][1]        # independent token batches
    assert all(res[r][2] for r in range(world))


def test_job_throughput_counts_all_ranks():
    import bench
    # 2 ranks x 10 steps x 4 units in 5 s of the slowest rank
    assert bench.job_throughput(4.0, 10, 2, 5.0) == pytest.approx(16.0)
    assert bench.max_over_ranks(None, [3.0, 1.0], "cpu") == [3.0, 1.0]
