"""pa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a plugin handed only its buffers, a server whose memory is all
reserved up front, a loop that cannot afford cudaMalloc's synchronisation).
Its split-KV scratch is a fixed-size array owned by the library, so this file
checks, through the C ABI, that it returns what pa_decode returns with a
caller workspace — on two calls in a row, so the second call runs on scratch
that still holds the first call's partials — and that a request too large for
the array is refused before anything is launched.

Kept last in collection order so that a failure here leaves the rest of the
GPU suite already run.
"""
import ctypes

import pytest
import torch

from paged_kv_cache_466_b200 import (KVPool, load_library, pa_decode, pa_decode_num_splits,
                                     pa_decode_workspace_bytes)
from paged_kv_cache_466_b200._lib import PA_ERR_WORKSPACE, PA_NOALLOC_SCRATCH_BYTES, PA_OK
from paged_kv_cache_466_b200 import workloads as W
from tests.helpers import DEV, device_append, device_inputs

pytestmark = pytest.mark.gpu
TOL = 1e-5        # the split-agreement tolerance of the decode tests


def _noalloc(lib, pool, q, bt, ctx, scale, out, num_splits):
    st = lib.pa_decode_noalloc(ctypes.byref(pool.c), ctypes.c_void_p(q.data_ptr()), q.shape[0],
                               q.shape[1], ctypes.c_void_p(bt.data_ptr()), bt.shape[1],
                               ctypes.c_void_p(ctx.data_ptr()), scale,
                               ctypes.c_void_p(out.data_ptr()), num_splits, None,
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def test_noalloc_matches_pa_decode_on_two_calls_in_a_row():
    # Both calls use at least two splits, so both run through the library's
    # array; the second one finds the first one's partials still there. The
    # computation is pa_decode's on different scratch, so the results must be
    # the same bits.
    lib = load_library()
    cases = [(W.llama8b(B=12, ctx_range=(100, 3000)), 8),
             (W.int8(B=6, ctx_range=(600, 900), seed=1), 3)]
    for w, splits in cases:
        pool, bt, ctx, q = device_inputs(w)
        device_append(pool, w, bt)
        S = pa_decode_num_splits(pool, w.B, w.max_pages, splits)
        assert S > 1, (w.name, S)
        assert pa_decode_workspace_bytes(w.B, w.Hq, w.D, S) <= PA_NOALLOC_SCRATCH_BYTES
        want = pa_decode(pool, q, bt, ctx, w.scale, num_splits=S)
        got = torch.full_like(want, float("nan"))
        assert _noalloc(lib, pool, q, bt, ctx, w.scale, got, S) == PA_OK
        torch.cuda.synchronize()
        err = (got - want).abs().max().item()
        assert err <= TOL, (w.name, S, err)
        assert torch.equal(got, want), (w.name, S)


def _shared_page_inputs(B, Hkv, Hq, max_pages, num_pages=2048, seed=0):
    """A bf16 pool of random pages and tables that draw their pages from it with
    repetition (decode only reads, so sequences may share pages): long tables
    at a small memory cost. Contexts span the whole table width."""
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    pool = KVPool(num_pages, Hkv, 16, 128, "bf16", DEV)
    for t in (pool.k, pool.v):
        t.copy_(torch.randn(t.shape, generator=g, device=DEV).to(torch.bfloat16))
    bt = torch.randint(0, num_pages, (B, max_pages), generator=g, device=DEV, dtype=torch.int32)
    ctx = torch.randint(1, max_pages * 16 + 1, (B,), generator=g, device=DEV, dtype=torch.int32)
    q = torch.randn((B, Hq, 128), generator=g, device=DEV).to(torch.bfloat16)
    return pool, bt, ctx, q


def test_noalloc_automatic_splits_fit_or_are_lowered():
    lib = load_library()
    # (1) a batch whose automatic plan already fits: same split count as pa_decode
    w = W.llama8b(B=12, ctx_range=(100, 3000), seed=2)
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    S = pa_decode_num_splits(pool, w.B, w.max_pages, 0)
    assert pa_decode_workspace_bytes(w.B, w.Hq, w.D, S) <= PA_NOALLOC_SCRATCH_BYTES
    want = pa_decode(pool, q, bt, ctx, w.scale, num_splits=0)
    got = torch.full_like(want, float("nan"))
    assert _noalloc(lib, pool, q, bt, ctx, w.scale, got, 0) == PA_OK
    torch.cuda.synchronize()
    assert torch.equal(got, want)

    # (2) a batch whose automatic plan needs more than the array holds: the
    # entry point takes the largest split count that fits instead. The
    # planner depends on the device's residency, so the batch is picked from a
    # few candidates as the first where that count is still above one.
    Hkv, Hq = 8, 48
    chosen = None
    for B, max_pages in ((256, 1024), (256, 2048), (384, 1024), (512, 512), (128, 2048)):
        probe = KVPool(1, Hkv, 16, 128, "bf16", DEV)
        S_auto = pa_decode_num_splits(probe, B, max_pages, 0)
        if pa_decode_workspace_bytes(B, Hq, 128, S_auto) <= PA_NOALLOC_SCRATCH_BYTES:
            continue
        S_fit = 1
        for s in range(S_auto - 1, 0, -1):
            Ss = pa_decode_num_splits(probe, B, max_pages, s)
            if pa_decode_workspace_bytes(B, Hq, 128, Ss) <= PA_NOALLOC_SCRATCH_BYTES:
                S_fit = Ss
                break
        if S_fit > 1:
            chosen = (B, max_pages, S_auto, S_fit)
            break
    assert chosen is not None, "no candidate batch needs its automatic split count lowered"
    B, max_pages, S_auto, S_fit = chosen
    pool, bt, ctx, q = _shared_page_inputs(B, Hkv, Hq, max_pages)
    scale = 128 ** -0.5
    want = pa_decode(pool, q, bt, ctx, scale, num_splits=S_fit)
    for _ in range(2):
        got = torch.full_like(want, float("nan"))
        assert _noalloc(lib, pool, q, bt, ctx, scale, got, 0) == PA_OK
        torch.cuda.synchronize()
        assert torch.equal(got, want), (chosen, (got - want).abs().max().item())


def test_noalloc_refuses_partials_larger_than_its_scratch():
    lib = load_library()
    w = W.llama8b(B=16, ctx_range=(3000, 4096))
    pool, bt, ctx, q = device_inputs(w)
    out = torch.zeros((w.B, w.Hq, w.D), dtype=torch.float32, device=DEV)
    S = pa_decode_num_splits(pool, w.B, w.max_pages, 256)
    assert pa_decode_workspace_bytes(w.B, w.Hq, w.D, S) > PA_NOALLOC_SCRATCH_BYTES
    assert _noalloc(lib, pool, q, bt, ctx, w.scale, out, 256) == PA_ERR_WORKSPACE
    assert b"scratch" in lib.pa_last_error()
    torch.cuda.synchronize()
    assert torch.all(out == 0)
