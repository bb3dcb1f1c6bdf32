"""The seeded input generators (shared by the oracle tests and the CUDA
tests; they hold none of the method's arithmetic): determinism, the page
recipe, and the per-sequence step-row layout pa_decode_append takes."""
import math

import numpy as np
import torch

from paged_kv_cache_466_b200 import workloads as W


def test_same_seed_same_inputs_and_tables():
    a, b = W.llama8b(B=5, ctx_range=(1, 300)), W.llama8b(B=5, ctx_range=(1, 300))
    assert np.array_equal(a.context_lens, b.context_lens)
    assert np.array_equal(a.block_tables, b.block_tables)
    assert torch.equal(a.q, b.q) and torch.equal(a.prefill_k, b.prefill_k)
    c = W.llama8b(B=5, ctx_range=(1, 300), seed=1)
    assert not torch.equal(a.q, c.q)


def test_tables_cover_each_context_with_distinct_pages():
    w = W.llama8b(B=9, ctx_range=(1, 2000))
    used = []
    for b in range(w.B):
        n = -(-int(w.context_lens[b]) // w.P)
        row = w.block_tables[b]
        assert np.all(row[:n] >= 0) and np.all(row[:n] < w.num_pages)
        assert np.all(row[n:] == -1)                      # never read, poisoned
        used += row[:n].tolist()
    assert len(used) == len(set(used))                   # no page owned twice
    assert w.num_pages == math.ceil(1.1 * len(used))     # the pool is need + 10 %


def test_rows_cover_every_position_once():
    w = W.paged("cov", B=4, Hq=4, Hkv=2, D=64, P=16, context_lens=[1, 16, 17, 40], kv="bf16")
    seq, pos, k, v = w.all_rows()
    got = sorted(zip(seq.tolist(), pos.tolist()))
    want = sorted((b, p) for b in range(w.B) for p in range(int(w.context_lens[b])))
    assert got == want
    assert k.shape == (len(seq), w.Hkv, w.D) and v.shape == k.shape


def test_step_rows_by_sequence_layout():
    w = W.paged("st", B=5, Hq=4, Hkv=2, D=64, P=16, context_lens=[3, 0, 17, 1, 32], kv="u8")
    k, v = w.step_rows_by_sequence()
    assert k.shape == (5, 2, 64) and k.dtype == torch.bfloat16
    for i, b in enumerate(w.step_seq.tolist()):
        assert int(w.step_pos[i]) == int(w.context_lens[b]) - 1
        assert torch.equal(k[b], w.step_k[i]) and torch.equal(v[b], w.step_v[i])
    assert torch.all(k[1] == 0) and torch.all(v[1] == 0)   # ctx 0: no step row
    # a step row that is not its sequence's newest position has no such layout
    w.step_pos = w.step_pos.copy()
    w.step_pos[0] -= 1
    assert w.step_rows_by_sequence() is None
