"""Test-side glue: move a seeded workload to the device through the library,
and build the oracle's own host pool from the same inputs."""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle
from paged_kv_cache_466_b200 import KVPool, pa_kv_append
from paged_kv_cache_466_b200.workloads import Workload, bits

DEV = "cuda"


def device_inputs(w: Workload, fill_byte: int = 0):
    pool = KVPool(w.num_pages, w.Hkv, w.P, w.D, w.kv, DEV, fill_byte=fill_byte)
    bt = torch.from_numpy(w.block_tables).to(DEV)
    ctx = torch.from_numpy(w.context_lens).to(DEV)
    q = w.q.to(DEV)
    return pool, bt, ctx, q


def device_append(pool: KVPool, w: Workload, bt: torch.Tensor, rows: str = "all",
                  d_err=None, chunk: int = 1 << 20):
    """Write the workload's prefill rows, then its step rows, with pa_kv_append."""
    parts = []
    if rows in ("all", "prefill"):
        parts.append((w.prefill_seq, w.prefill_pos, w.prefill_k, w.prefill_v))
    if rows in ("all", "step"):
        parts.append((w.step_seq, w.step_pos, w.step_k, w.step_v))
    for seq, pos, k, v in parts:
        for a in range(0, len(seq), chunk):
            b = min(a + chunk, len(seq))
            if b <= a:
                continue
            pa_kv_append(pool, k[a:b].to(DEV), v[a:b].to(DEV),
                         torch.from_numpy(seq[a:b]).to(DEV), torch.from_numpy(pos[a:b]).to(DEV),
                         bt, d_err=d_err)


def oracle_pool(w: Workload, fill_byte: int = 0) -> oracle.HostPool:
    hp = oracle.empty_pool(w.kv, w.num_pages, w.Hkv, w.P, w.D, fill_byte)
    oracle.scatter_rows(hp, w.block_tables, w.prefill_seq, w.prefill_pos,
                        bits(w.prefill_k), bits(w.prefill_v))
    oracle.scatter_rows(hp, w.block_tables, w.step_seq, w.step_pos,
                        bits(w.step_k), bits(w.step_v))
    return hp


def oracle_decode(w: Workload, hp: oracle.HostPool, pairs=None):
    out, lse = oracle.paged_attention(hp, bits(w.q), w.block_tables, w.context_lens, w.scale,
                                      pairs=pairs)
    return out, lse


def pool_bytes_equal(pool: KVPool, hp: oracle.HostPool):
    """Byte-for-byte comparison of the device pool with the oracle's pool."""
    pairs = [(pool.k, hp.k), (pool.v, hp.v)]
    if hp.kind in ("u8", "fp8", "u4"):
        pairs += [(pool.k_sz, hp.k_sz), (pool.v_sz, hp.v_sz)]
    for dt, ht in pairs:
        got = dt.view(torch.uint8).cpu().numpy().reshape(-1)
        want = ht.view(np.uint8).reshape(-1)
        if not np.array_equal(got, want):
            bad = np.flatnonzero(got != want)
            return False, f"{bad.size} bytes differ, first at byte {bad[0]}"
    return True, ""


@functools.lru_cache(maxsize=8)
def full_size_reference(name: str):
    """The named full-size workload with the oracle's pool and its fp64 Eq. 1
    output for every (sequence, query head) row, computed once per test
    process (the larger workloads take seconds on the host)."""
    from paged_kv_cache_466_b200 import workloads as W
    w = W.by_name(name)
    hp = oracle_pool(w)
    ref, lse = oracle_decode(w, hp)
    return w, ref, lse
