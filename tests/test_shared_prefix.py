"""pa_decode_shared_prefix (cascade decode over a shared prompt prefix) on the
GPU: it must equal the fp64 oracle of Eq. 1 over the full contexts (2e-3, the
decode tolerance) and agree with the plain paged decode of the same tables."""
import numpy as np
import pytest
import torch

from paged_kv_cache_466_b200 import (pa_decode, pa_decode_shared_prefix,
                                     pa_decode_shared_prefix_workspace_bytes, pa_kv_append)
from paged_kv_cache_466_b200 import workloads as W
from tests.helpers import (DEV, device_append, device_inputs, full_size_reference,
                           oracle_decode, oracle_pool)

pytestmark = pytest.mark.gpu


def _both(w, num_splits=0, ctx_override=None):
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    if ctx_override is not None:
        ctx = torch.from_numpy(ctx_override).to(DEV)
    pre = torch.from_numpy(np.ascontiguousarray(w.notes["prefix_pages"])).to(DEV)
    casc = pa_decode_shared_prefix(pool, q, pre, w.notes["prefix_tokens"], bt, ctx, w.scale,
                                   num_splits=num_splits)
    plain = pa_decode(pool, q, bt, ctx, w.scale)
    torch.cuda.synchronize()
    return casc.cpu().numpy().reshape(-1, w.D), plain.cpu().numpy().reshape(-1, w.D)


@pytest.mark.parametrize("kw", [
    dict(B=8, prefix_tokens=64, suffix_range=(1, 50)),
    dict(B=5, prefix_tokens=160, suffix_range=(1, 300), Hq=8, Hkv=2),          # 20 query rows
    dict(B=7, prefix_tokens=192, suffix_range=(1, 100), Hq=16, Hkv=2, P=32),   # G = 8, P = 32
    dict(B=6, prefix_tokens=96, suffix_range=(1, 40), Hq=4, Hkv=4, D=64),      # G = 1, D = 64
    dict(B=33, prefix_tokens=1008, suffix_range=(1, 20)),                      # ragged last tile
], ids=["small", "rows20", "g8-p32", "d64-g1", "ragged-tile"])
@pytest.mark.parametrize("num_splits", [0, 1, 4])
def test_cascade_matches_oracle_and_plain_decode(kw, num_splits):
    w, _ = W.prefix(**kw)
    casc, plain = _both(w, num_splits)
    ref, _ = oracle_decode(w, oracle_pool(w))
    err = np.abs(casc - ref).max()
    print(f"cascade {kw}: max |gpu - oracle| = {err:.3e}, vs plain {np.abs(casc - plain).max():.3e}")
    assert np.all(np.isfinite(casc)) and err <= 2e-3
    assert np.abs(casc - plain).max() <= 1e-4


def test_cascade_requests_without_own_tokens():
    """ctx == prefix_len: the output is the prefix attention alone."""
    w, _ = W.prefix(B=6, prefix_tokens=128, suffix_range=(1, 60))
    ctx = w.context_lens.copy()
    ctx[[0, 3]] = 128
    casc, plain = _both(w, ctx_override=ctx)
    w.context_lens = ctx
    ref, _ = oracle_decode(w, oracle_pool(w))
    assert np.abs(casc - ref).max() <= 2e-3
    assert np.abs(casc - plain).max() <= 1e-4


def test_cascade_full_size_prefix_workload():
    """128 requests x (2000-token shared prefix + U{1..512} own tokens): every
    row against the oracle and against the plain paged decode."""
    w, ref, _ = full_size_reference("prefix")
    casc, plain = _both(w)
    err = np.abs(casc - ref).max()
    print(f"cascade full size: all {ref.shape[0]} rows, max |gpu - oracle| = {err:.3e}")
    assert np.all(np.isfinite(casc)) and err <= 2e-3
    assert np.abs(casc - plain).max() <= 1e-4


def test_cascade_reads_rows_appended_just_before_it():
    """The suffix decode skips its own programmatic wait (only the prefix pass
    waits for the work before the call): rows that pa_kv_append writes right
    before the call, on the same stream with nothing between, must still be
    read. Unwritten slots hold the byte 0xFF (bf16 NaN), so a read that beat
    the append would show; the suffixes are a few tokens, the newest one a
    large part of each."""
    w, _ = W.prefix(B=24, prefix_tokens=128, suffix_range=(1, 6))
    pool, bt, ctx, q = device_inputs(w, fill_byte=0xFF)
    pre = torch.from_numpy(np.ascontiguousarray(w.notes["prefix_pages"])).to(DEV)
    ref, _ = oracle_decode(w, oracle_pool(w))
    sk, sv = w.step_k.to(DEV), w.step_v.to(DEV)
    sseq, spos = torch.from_numpy(w.step_seq).to(DEV), torch.from_numpy(w.step_pos).to(DEV)
    for it in range(3):
        for t in (pool.k, pool.v):
            t.view(torch.uint8).fill_(0xFF)
        device_append(pool, w, bt, rows="prefill")
        torch.cuda.synchronize()
        pa_kv_append(pool, sk, sv, sseq, spos, bt)  # the newest rows, then at once:
        out = pa_decode_shared_prefix(pool, q, pre, w.notes["prefix_tokens"], bt, ctx, w.scale)
        torch.cuda.synchronize()
        got = out.cpu().numpy().reshape(-1, w.D)
        assert np.all(np.isfinite(got)), f"call {it}: a row was read before the append wrote it"
        err = np.abs(got - ref).max()
        assert err <= 2e-3, f"call {it}: max |gpu - oracle| = {err:.3e}"


def test_cascade_captured_in_a_cuda_graph_replays_the_eager_bits():
    """Called eagerly, the prefix pass, the suffix decode and the merge are one
    chain of programmatic launches on the caller's stream; captured in a CUDA
    graph, the suffix decode is a branch forked from and joined back to it.
    The graph replays to the eager call's bits, twice in a row."""
    w, _ = W.prefix(B=33, prefix_tokens=1008, suffix_range=(1, 200))
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    pre = torch.from_numpy(np.ascontiguousarray(w.notes["prefix_pages"])).to(DEV)
    eager = pa_decode_shared_prefix(pool, q, pre, w.notes["prefix_tokens"], bt, ctx, w.scale)
    torch.cuda.synchronize()
    out = torch.zeros_like(eager)
    need = pa_decode_shared_prefix_workspace_bytes(pool, w.B, w.Hq, bt.shape[1],
                                                   w.notes["prefix_tokens"], 0)
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    pa_decode_shared_prefix(pool, q, pre, w.notes["prefix_tokens"], bt, ctx, w.scale, out=out,
                            workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pa_decode_shared_prefix(pool, q, pre, w.notes["prefix_tokens"], bt, ctx, w.scale,
                                out=out, workspace=ws)
    for _ in range(2):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    ref, _ = oracle_decode(w, oracle_pool(w))
    assert np.abs(out.cpu().numpy().reshape(-1, w.D) - ref).max() <= 2e-3


def test_cascade_from_two_host_threads_on_two_streams():
    """Two host threads run the cascade on their own streams, over the same
    batch with their own outputs and workspaces, many calls each: every output
    equals the single-thread result bit for bit (each call's launches stay
    inside its own stream's order)."""
    import threading
    w, _ = W.prefix(B=20, prefix_tokens=320, suffix_range=(1, 120))
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    pre = torch.from_numpy(np.ascontiguousarray(w.notes["prefix_pages"])).to(DEV)
    want = pa_decode_shared_prefix(pool, q, pre, w.notes["prefix_tokens"], bt, ctx, w.scale)
    torch.cuda.synchronize()
    need = pa_decode_shared_prefix_workspace_bytes(pool, w.B, w.Hq, bt.shape[1],
                                                   w.notes["prefix_tokens"], 0)
    errors = []

    def worker():
        try:
            s = torch.cuda.Stream()
            out = torch.zeros_like(want)
            ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
            with torch.cuda.stream(s):
                for _ in range(50):
                    pa_decode_shared_prefix(pool, q, pre, w.notes["prefix_tokens"], bt, ctx,
                                            w.scale, out=out, workspace=ws, stream=s)
            s.synchronize()
            if not torch.equal(out, want):
                errors.append("mismatch")
        except Exception as e:  # pragma: no cover - reported below
            errors.append(repr(e))

    threads = [threading.Thread(target=worker) for _ in range(2)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
