"""Failure detection on the GPU without a fault: a bounded wait that can
never be satisfied ends with PA_DERR_TIMEOUT in the error word, within its
time limit, and the context keeps working afterwards."""
import time

import pytest
import torch

from paged_kv_cache_466_b200 import (PA_DERR_TIMEOUT, pa_decode, pa_derr_status,
                                     pa_selftest_wait_timeout)
from paged_kv_cache_466_b200 import _lib
from paged_kv_cache_466_b200 import workloads as W
from tests.helpers import DEV, device_append, device_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_us", [50, 2000, 20000])
def test_unsatisfiable_wait_times_out_and_context_survives(limit_us):
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    pa_selftest_wait_timeout(limit_us, err)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    e = int(err.item())
    assert e == PA_DERR_TIMEOUT
    assert pa_derr_status(e) == _lib.PA_ERR_TIMEOUT
    assert limit_us * 1e-6 <= dt < limit_us * 1e-6 + 0.5
    # the context is still usable: a decode runs and is correct-shaped
    w = W.tiny()
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    out = pa_decode(pool, q, bt, ctx, w.scale)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
