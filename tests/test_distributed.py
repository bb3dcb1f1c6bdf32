"""The multi-GPU bench path on CPU: two gloo ranks. The decode shards into
independent sequences, so the only cross-rank steps are the timing barrier and
the max over ranks; each rank draws its own seeded batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 7.5][rank]
        m = bench.max_over_ranks(ms, world)
        dist.barrier()
        w = bench.make_workload("tiny", seed=rank)
        q.put((rank, m, bench.whole_job_gbs(1_000_000, world, m),
               w.q.float().sum().item(), w.block_tables.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, v0, s0, t0), (r1, m1, v1, s1, t1) = res
    assert m0 == m1 == 7.5                       # both ranks see the slowest rank
    assert v0 == v1 == pytest.approx(2 * 1_000_000 / 7.5e-3 / 1e9)
    assert s0 != s1                              # different seeded shards per rank


def test_single_rank_passthrough():
    assert bench.max_over_ranks(4.25, 1) == 4.25
    assert bench.whole_job_gbs(2_000_000_000, 1, 1.0) == pytest.approx(2000.0)
