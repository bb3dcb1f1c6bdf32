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


def _cp_worker(rank, world, port, q):
    """One rank of a context-parallel decode with the oracle standing in for
    pa_decode_range: partial over this rank's token range, written into this
    rank's block of the packed layout decode_context_parallel gathers, one
    all-gather, merge of the strided views."""
    import oracle
    from paged_kv_cache_466_b200 import workloads as W
    from paged_kv_cache_466_b200.context_parallel import (gathered_views, partial_block_floats,
                                                           partial_views, rank_range)
    from paged_kv_cache_466_b200.workloads import bits
    from tests.helpers import oracle_pool
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.paged("cp", B=3, Hq=4, Hkv=2, D=64, P=16, context_lens=[5, 70, 200], kv="bf16")
        hp = oracle_pool(w)
        b, e = rank_range(rank, world, 64)
        o, lse = oracle.paged_attention(hp, bits(w.q), w.block_tables, w.context_lens, w.scale,
                                        t_begin=b, t_end=e if e < 0x7FFFFFFF else -1)
        block = torch.full((partial_block_floats(w.B, w.Hq, w.D),), float("nan"))
        ov, lv = partial_views(block, w.B, w.Hq, w.D)
        ov.copy_(torch.from_numpy(o).view(w.B, w.Hq, w.D))
        lv.copy_(torch.from_numpy(lse).view(w.B, w.Hq))
        gathered = torch.empty(world * block.numel())
        dist.all_gather_into_tensor(gathered, block)
        o_parts, l_parts = gathered_views(gathered, world, w.B, w.Hq, w.D)
        merged = oracle.lse_merge(o_parts.double().numpy().reshape(world, -1, w.D).transpose(1, 0, 2),
                                  l_parts.double().numpy().reshape(world, -1).T)
        full, _ = oracle.paged_attention(hp, bits(w.q), w.block_tables, w.context_lens, w.scale)
        # fp32 partials: the merge of the rounded parts is within fp32 rounding of Eq. 1
        q.put((rank, float(np.abs(merged - full).max())))
    finally:
        dist.destroy_process_group()


def test_context_parallel_ranges_merge_to_the_full_decode():
    """Three gloo ranks, 64 tokens each (the last one open-ended): the merged
    range partials equal Eq. 1 over the whole contexts, which shows that the
    ranges cover every token once and that the part-major gather is merged
    with the right weights."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, 3, port, q)) for r in range(3)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, err in res:
        assert err <= 1e-6


def test_rank_ranges():
    from paged_kv_cache_466_b200.context_parallel import rank_range
    assert [rank_range(r, 3, 32) for r in range(3)] == [(0, 32), (32, 64), (64, 0x7FFFFFFF)]
    assert rank_range(0, 1, 16) == (0, 0x7FFFFFFF)
    with pytest.raises(ValueError):
        rank_range(3, 3, 32)


def test_packed_partial_layout():
    """Each rank's block holds o then lse, 256-byte aligned; the gathered
    views see rank r's values in part r."""
    from paged_kv_cache_466_b200.context_parallel import (gathered_views, partial_block_floats,
                                                           partial_views)
    B, Hq, D, world = 3, 5, 12, 4
    n = partial_block_floats(B, Hq, D)
    assert n % 64 == 0 and n >= B * Hq * (D + 1)
    gathered = torch.zeros(world * n)
    for r in range(world):
        o, lse = partial_views(gathered[r * n:(r + 1) * n], B, Hq, D)
        o.copy_(torch.arange(B * Hq * D, dtype=torch.float32).view(B, Hq, D) + 1000 * r)
        lse.copy_(torch.arange(B * Hq, dtype=torch.float32).view(B, Hq) - 1000 * r)
    o_parts, l_parts = gathered_views(gathered, world, B, Hq, D)
    assert o_parts.shape == (world, B, Hq, D) and l_parts.shape == (world, B, Hq)
    assert o_parts.stride(0) == n and l_parts.stride(0) == n and o_parts[0].is_contiguous()
    for r in range(world):
        assert torch.equal(o_parts[r].flatten(), torch.arange(B * Hq * D, dtype=torch.float32) + 1000 * r)
        assert torch.equal(l_parts[r].flatten(), torch.arange(B * Hq, dtype=torch.float32) - 1000 * r)


def _cp_api_worker(rank, world, port, q):
    """decode_context_parallel itself on gloo ranks, with the two library calls
    replaced by the oracle (same signatures, same output buffers): checks the
    packing, the single all-gather and the strided merge views end to end."""
    import types
    import oracle
    from paged_kv_cache_466_b200 import context_parallel as cp
    from paged_kv_cache_466_b200 import workloads as W
    from paged_kv_cache_466_b200.workloads import bits
    from tests.helpers import oracle_pool
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.paged("cpapi", B=4, Hq=8, Hkv=2, D=64, P=16, context_lens=[1, 40, 130, 300],
                    kv="u8")
        hp = oracle_pool(w)
        calls = []

        def fake_range(pool, qq, bt, ctx, scale, b, e, o_out=None, lse_out=None, **kw):
            calls.append((b, e))
            o, l = oracle.paged_attention(pool.hp, bits(qq), bt.numpy(), ctx.numpy(), scale,
                                          t_begin=b, t_end=e if e < 0x7FFFFFFF else -1)
            o_out.copy_(torch.from_numpy(o).view(o_out.shape))
            lse_out.copy_(torch.from_numpy(l).view(lse_out.shape))
            return o_out, lse_out

        def fake_merge(o_parts, lse_parts, out=None, lse_out=None, stream=None):
            n, D = o_parts.shape[0], o_parts.shape[-1]
            m = oracle.lse_merge(o_parts.double().numpy().reshape(n, -1, D).transpose(1, 0, 2),
                                 lse_parts.double().numpy().reshape(n, -1).T)
            res = torch.from_numpy(m).float().view(o_parts.shape[1:])
            if out is not None:
                out.copy_(res)
                res = out
            return res, None

        cp.pa_decode_range, cp.pa_merge_partials = fake_range, fake_merge
        pool = types.SimpleNamespace(page_size=w.P, hp=hp)
        out = cp.decode_context_parallel(pool, w.q, torch.from_numpy(w.block_tables),
                                         torch.from_numpy(w.context_lens), w.scale,
                                         tokens_per_rank=64)
        full, _ = oracle.paged_attention(hp, bits(w.q), w.block_tables, w.context_lens, w.scale)
        err = float(np.abs(out.double().numpy().reshape(-1, w.D) - full).max())
        q.put((rank, calls, err))
    finally:
        dist.destroy_process_group()


def test_decode_context_parallel_orchestration_on_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_cp_api_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [[(0, 64)], [(64, 128)], [(128, 0x7FFFFFFF)]]
    for _, _, err in res:
        assert err <= 1e-6


def _cp_bench_worker(rank, world, port, q):
    """The bench's context-parallel mode on gloo ranks: each rank builds its
    own pool from bench.cp_shard_rows (its token range of the same seeded
    batch, its own page ids) and runs decode_context_parallel with the oracle
    standing in for the two library calls."""
    import types
    import oracle
    from paged_kv_cache_466_b200 import context_parallel as cp
    from paged_kv_cache_466_b200 import workloads as W
    from paged_kv_cache_466_b200.workloads import bits
    from tests.helpers import oracle_pool
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.paged("cpbench", B=5, Hq=8, Hkv=2, D=64, P=16, ctx_range=(1, 300), kv="bf16",
                    seed=3)
        T, (begin, end), tables, n_pages, (seq, pos, k, v) = bench.cp_shard_rows(w, rank, world)
        hp = oracle.empty_pool(w.kv, n_pages, w.Hkv, w.P, w.D, 0xFF)   # NaN-ish filler
        oracle.scatter_rows(hp, tables, seq, pos, bits(k), bits(v))

        def fake_range(pool, qq, bt, ctx, scale, b, e, o_out=None, lse_out=None, **kw):
            o, l = oracle.paged_attention(pool.hp, bits(qq), bt.numpy(), ctx.numpy(), scale,
                                          t_begin=b, t_end=e if e < 0x7FFFFFFF else -1)
            o_out.copy_(torch.from_numpy(o).view(o_out.shape))
            lse_out.copy_(torch.from_numpy(l).view(lse_out.shape))
            return o_out, lse_out

        def fake_merge(o_parts, lse_parts, out=None, lse_out=None, stream=None):
            n, D = o_parts.shape[0], o_parts.shape[-1]
            m = oracle.lse_merge(o_parts.double().numpy().reshape(n, -1, D).transpose(1, 0, 2),
                                 lse_parts.double().numpy().reshape(n, -1).T)
            res = torch.from_numpy(m).float().view(o_parts.shape[1:])
            out.copy_(res)
            return out, None

        cp.pa_decode_range, cp.pa_merge_partials = fake_range, fake_merge
        pool = types.SimpleNamespace(page_size=w.P, hp=hp)
        out = torch.empty((w.B, w.Hq, w.D))
        cp.decode_context_parallel(pool, w.q, torch.from_numpy(tables),
                                   torch.from_numpy(w.context_lens), w.scale, T, out=out)
        full, _ = oracle.paged_attention(oracle_pool(w), bits(w.q), w.block_tables,
                                         w.context_lens, w.scale)
        err = float(np.abs(out.double().numpy().reshape(-1, w.D) - full).max())
        own = int(sum(max(0, min(int(c), end) - begin) for c in w.context_lens))
        q.put((rank, T, len(seq), own, n_pages, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_bench_context_parallel_shards_merge_to_the_full_decode(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_bench_worker, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from paged_kv_cache_466_b200 import workloads as W
    w = W.paged("cpbench", B=5, Hq=8, Hkv=2, D=64, P=16, ctx_range=(1, 300), kv="bf16", seed=3)
    assert sum(r[2] for r in res) == w.total_tokens       # every row on exactly one rank
    for _, T, nrows, own, n_pages, err in res:
        assert T % w.P == 0 and nrows == own
        assert n_pages >= -(-own // w.P)
        assert err <= 1e-6
