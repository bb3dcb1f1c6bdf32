"""pa_decode_range and pa_merge_partials on one GPU: the shards of a
context-parallel decode computed one after another (no collective needed to
check the arithmetic) and merged; they must equal the single-GPU decode and
the fp64 oracle."""
import numpy as np
import pytest
import torch

from paged_kv_cache_466_b200 import pa_decode, pa_decode_range, pa_merge_partials
from paged_kv_cache_466_b200 import workloads as W
from paged_kv_cache_466_b200.context_parallel import (gathered_views, partial_block_floats,
                                                       partial_views, rank_range)
from paged_kv_cache_466_b200.workloads import bits
import oracle
from tests.helpers import DEV, device_append, device_inputs, oracle_pool

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.mark.parametrize("kv", ["bf16", "u8", "fp8", "u4"])
@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_range_partials_match_the_oracle(kv, num_splits):
    w = W.paged("rng", B=5, Hq=8, Hkv=2, D=128, P=16, context_lens=[1, 40, 300, 700, 33], kv=kv)
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    hp = oracle_pool(w)
    for b, e in [(0, 64), (32, 500), (304, 0x7FFFFFFF), (640, 700), (48, 48)]:
        o, lse = pa_decode_range(pool, q, bt, ctx, w.scale, b, e, num_splits=num_splits)
        torch.cuda.synchronize()
        ro, rl = oracle.paged_attention(hp, bits(w.q), w.block_tables, w.context_lens, w.scale,
                                        t_begin=b, t_end=-1 if e >= 0x7FFFFFFF else e)
        o = o.cpu().numpy().reshape(-1, w.D)
        lse = lse.cpu().numpy().reshape(-1)
        assert np.all(np.isfinite(o))
        assert np.abs(o - ro).max() <= TOL
        empty = ~np.isfinite(rl)
        assert np.all(np.isneginf(lse[empty])) and np.all(o[empty] == 0)
        if (~empty).any():
            assert np.abs(lse[~empty] - rl[~empty]).max() <= 1e-4


@pytest.mark.parametrize("world,tpr", [(2, 256), (3, 128), (4, 64)])
def test_emulated_ranks_merge_to_the_single_gpu_decode(world, tpr):
    w = W.llama8b(B=6, ctx_range=(1, 900))
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    parts = [pa_decode_range(pool, q, bt, ctx, w.scale, *rank_range(r, world, tpr))
             for r in range(world)]
    o_all = torch.stack([p[0] for p in parts])
    l_all = torch.stack([p[1] for p in parts])
    out, lse = pa_merge_partials(o_all, l_all)
    full = pa_decode(pool, q, bt, ctx, w.scale)
    torch.cuda.synchronize()
    assert (out - full).abs().max().item() <= 5e-5
    ref, rl = oracle.paged_attention(oracle_pool(w), bits(w.q), w.block_tables, w.context_lens,
                                     w.scale)
    assert np.abs(out.cpu().numpy().reshape(-1, w.D) - ref).max() <= TOL
    assert np.abs(lse.cpu().numpy().reshape(-1) - rl).max() <= 1e-4


@pytest.mark.parametrize("kv", ["bf16", "u8"])
def test_emulated_ranks_in_the_packed_gather_layout(kv):
    """What decode_context_parallel does on each rank, minus the collective:
    every rank's range decode writes o and lse into its own block of one
    buffer (the all-gather's output layout) and the merge reads the strided
    views in place."""
    world, tpr = 3, 96
    w = W.paged("pk", B=7, Hq=16, Hkv=2, D=128, P=32, ctx_range=(1, 700), kv=kv)
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    n = partial_block_floats(w.B, w.Hq, w.D)
    gathered = torch.full((world * n,), float("nan"), device=DEV)
    for r in range(world):
        o, lse = partial_views(gathered[r * n:(r + 1) * n], w.B, w.Hq, w.D)
        pa_decode_range(pool, q, bt, ctx, w.scale, *rank_range(r, world, tpr), o_out=o,
                        lse_out=lse)
    o_parts, l_parts = gathered_views(gathered, world, w.B, w.Hq, w.D)
    out, lse = pa_merge_partials(o_parts, l_parts)
    full = pa_decode(pool, q, bt, ctx, w.scale)
    torch.cuda.synchronize()
    assert (out - full).abs().max().item() <= 5e-5
    ref, rl = oracle.paged_attention(oracle_pool(w), bits(w.q), w.block_tables, w.context_lens,
                                     w.scale)
    assert np.abs(out.cpu().numpy().reshape(-1, w.D) - ref).max() <= TOL


def test_merge_rejects_overlapping_parts():
    o = torch.zeros(3, 4, 8, device=DEV)
    l = torch.zeros(3, 4, device=DEV)
    with pytest.raises(ValueError):
        pa_merge_partials(o.view(-1)[:24 * 4].as_strided((3, 4, 8), (16, 8, 1)), l)


def test_merge_partials_against_the_oracle_merge():
    g = torch.Generator().manual_seed(7)
    n, rows, D = 5, 37, 64
    o = torch.randn(n, rows, D, generator=g)
    lse = torch.randn(n, rows, generator=g) * 3
    lse[:2, 0] = -float("inf")
    lse[:, 1] = -float("inf")                           # every part empty: 0, -inf
    out, lo = pa_merge_partials(o.to(DEV), lse.to(DEV))
    want = oracle.lse_merge(o.double().numpy().transpose(1, 0, 2), lse.double().numpy().T)
    assert np.abs(out.cpu().numpy() - want).max() <= 1e-5
    assert torch.all(out[1] == 0) and torch.isneginf(lo[1]).item()
    m = np.max(lse.double().numpy(), axis=0)
    fin = np.isfinite(m)
    wl = np.log(np.sum(np.exp(lse.double().numpy()[:, fin] - m[fin]), axis=0)) + m[fin]
    assert np.abs(lo.cpu().numpy()[fin] - wl).max() <= 1e-5


@pytest.mark.parametrize("world", [1, 2, 3])
def test_bench_shards_decoded_per_rank_merge_to_the_oracle(world):
    """The bench's context-parallel layout on one GPU: every emulated rank
    gets its own pool and tables from bench.cp_shard_rows, decodes its token
    range, and the packed partials merge to Eq. 1 over the whole contexts.
    With one rank decode_context_parallel itself runs (no process group)."""
    import bench
    from paged_kv_cache_466_b200 import KVPool, pa_kv_append
    from paged_kv_cache_466_b200.context_parallel import decode_context_parallel
    w = W.llama8b(B=5, ctx_range=(1, 1500), seed=11)
    ref, _ = oracle.paged_attention(oracle_pool(w), bits(w.q), w.block_tables, w.context_lens,
                                    w.scale)
    q = w.q.to(DEV)
    ctx = torch.from_numpy(w.context_lens).to(DEV)
    n = partial_block_floats(w.B, w.Hq, w.D)
    gathered = torch.full((world * n,), float("nan"), device=DEV)
    for r in range(world):
        T, (b, e), tables, n_pages, (seq, pos, k, v) = bench.cp_shard_rows(w, r, world)
        pool = KVPool(n_pages, w.Hkv, w.P, w.D, w.kv, DEV, fill_byte=0xFF)
        bt = torch.from_numpy(tables).to(DEV)
        pa_kv_append(pool, k.to(DEV), v.to(DEV), torch.from_numpy(seq).to(DEV),
                     torch.from_numpy(pos).to(DEV), bt)
        if world == 1:
            out = decode_context_parallel(pool, q, bt, ctx, w.scale, T)
            break
        o, lse = partial_views(gathered[r * n:(r + 1) * n], w.B, w.Hq, w.D)
        pa_decode_range(pool, q, bt, ctx, w.scale, b, e, o_out=o, lse_out=lse)
    if world > 1:
        o_parts, l_parts = gathered_views(gathered, world, w.B, w.Hq, w.D)
        out, _ = pa_merge_partials(o_parts, l_parts)
    torch.cuda.synchronize()
    assert np.abs(out.cpu().numpy().reshape(-1, w.D) - ref).max() <= TOL
