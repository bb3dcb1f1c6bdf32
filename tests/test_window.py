"""pa_decode_window (attention sinks + sliding window, Eq. 5 / Eq. 6) on the GPU
against the fp64 oracle of the same token set, with the evicted pages poisoned
to show they are never read."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_466_b200 import pa_decode, pa_decode_window
from paged_kv_cache_466_b200 import workloads as W
from paged_kv_cache_466_b200.workloads import bits
from tests.helpers import DEV, device_append, device_inputs, oracle_pool

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _evicted_pages(w, sinks, window):
    ev = []
    for b in range(w.B):
        n = int(w.context_lens[b])
        keep = np.zeros(n, bool)
        keep[:min(sinks, n)] = True
        keep[max(n - window, 0):] = True
        for lp in range(-(-n // w.P)):
            if not keep[lp * w.P:(lp + 1) * w.P].any():
                ev.append(int(w.block_tables[b, lp]))
    return ev


def _run(w, sinks, window, num_splits=0, poison=True):
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    if poison:
        ev = torch.tensor(_evicted_pages(w, sinks, window), dtype=torch.long, device=DEV)
        if ev.numel():
            for t in pool.tensors():
                t.view(torch.uint8)[ev] = 0xFF       # NaN in bf16 and fp32
    out = pa_decode_window(pool, q, bt, ctx, w.scale, sinks, window, num_splits=num_splits)
    torch.cuda.synchronize()
    return out.cpu().numpy().reshape(-1, w.D)


CASES = {
    "bf16-p16": lambda: W.llama8b(B=6, ctx_range=(1, 900)),
    "bf16-p32-g8": lambda: W.paged("p32", B=4, Hq=32, Hkv=4, D=128, P=32, ctx_range=(1, 1200)),
    "int8": lambda: W.int8(B=6, ctx_range=(1, 900)),
    "d64": lambda: W.paged("d64", B=5, Hq=8, Hkv=2, D=64, P=16, ctx_range=(1, 400)),
    "fp8": lambda: W.fp8(B=6, ctx_range=(1, 900)),
    "int4": lambda: W.int4(B=6, ctx_range=(1, 900)),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("sinks,window", [(0, 1), (0, 37), (4, 100), (4, 256), (16, 33),
                                          (1000, 50), (3, 5000)])
def test_window_matches_oracle(name, sinks, window):
    w = CASES[name]()
    got = _run(w, sinks, window)
    ref, _ = oracle.paged_attention_window(oracle_pool(w), bits(w.q), w.block_tables,
                                           w.context_lens, w.scale, sinks, window)
    err = np.abs(got - ref).max()
    print(f"{name} s={sinks} w={window}: max |gpu - oracle| = {err:.3e}")
    assert np.all(np.isfinite(got)) and err <= TOL


@pytest.mark.parametrize("num_splits", [1, 2, 5])
def test_window_split_counts_agree(num_splits):
    w = W.llama70b(B=3, ctx=3000)
    a = _run(w, 4, 1500, num_splits=0)
    b = _run(w, 4, 1500, num_splits=num_splits)
    assert np.abs(a - b).max() <= 1e-5


def test_window_of_one_is_the_newest_value_row():
    w = W.paged("w1", B=4, Hq=16, Hkv=2, D=128, P=16, ctx_range=(1, 300))
    got = _run(w, 0, 1)
    last = np.stack([w.step_v[i].float().numpy() for i in range(w.B)])   # [B, Hkv, D]
    want = np.repeat(last, w.G, axis=1).reshape(-1, w.D)
    np.testing.assert_array_equal(got, want)


def test_window_covering_the_context_equals_plain_decode():
    w = W.llama8b(B=5, ctx_range=(1, 700))
    got = _run(w, 0, 4096, poison=False)
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    plain = pa_decode(pool, q, bt, ctx, w.scale).cpu().numpy().reshape(-1, w.D)
    assert np.abs(got - plain).max() <= 1e-5


@pytest.mark.parametrize("name", ["bf16-p16", "int8", "int4"])
@pytest.mark.parametrize("num_splits", [2, 3])
def test_window_sinks_share_the_first_split(name, num_splits):
    """The sinks are a second token range of split 0 (no split of their own):
    with forced splits, ragged contexts put sequences where split 0 holds only
    sinks, sinks plus window tokens, or where later splits are empty; every
    row equals the oracle's Eq. 5 over exactly the kept tokens."""
    w = CASES[name]()
    for sinks, window in ((16, 40), (5, 300), (40, 17)):
        got = _run(w, sinks, window, num_splits=num_splits)
        ref, _ = oracle.paged_attention_window(oracle_pool(w), bits(w.q), w.block_tables,
                                               w.context_lens, w.scale, sinks, window)
        err = np.abs(got - ref).max()
        assert np.all(np.isfinite(got)) and err <= TOL, (sinks, window, err)
