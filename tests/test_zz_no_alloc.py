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

import numpy as np
import pytest
import torch

from paged_kv_cache_466_b200 import (PagedAttnError, load_library, pa_decode,
                                     pa_decode_num_splits, pa_decode_workspace_bytes)
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
    lib = load_library()
    cases = [(W.llama8b(B=12, ctx_range=(100, 3000)), 8),
             (W.int8(B=6, ctx_range=(1, 900), seed=1), 0)]
    for w, splits in cases:
        pool, bt, ctx, q = device_inputs(w)
        device_append(pool, w, bt)
        S = pa_decode_num_splits(pool, w.B, w.max_pages, splits)
        assert pa_decode_workspace_bytes(w.B, w.Hq, w.D, S) <= PA_NOALLOC_SCRATCH_BYTES
        want = pa_decode(pool, q, bt, ctx, w.scale, num_splits=S)
        got = torch.full_like(want, float("nan"))
        assert _noalloc(lib, pool, q, bt, ctx, w.scale, got, S) == PA_OK
        torch.cuda.synchronize()
        err = (got - want).abs().max().item()
        assert err <= TOL, (w.name, S, err)
        assert S > 1 or splits == 0


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
