"""pa_decode_append: the newest token's cache write fused into the decode. It
must store exactly what pa_kv_append stores (the whole pool byte for byte
against the oracle's scatter and quantiser) and return exactly what
pa_kv_append followed by pa_decode returns, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_466_b200 import pa_decode, pa_decode_append
from paged_kv_cache_466_b200 import workloads as W
from paged_kv_cache_466_b200.workloads import bits
from tests.helpers import (DEV, device_append, device_inputs, full_size_reference, oracle_pool,
                           pool_bytes_equal)

pytestmark = pytest.mark.gpu
RAGGED = [0, 1, 5000, 17, 0, 3, 16, 32, 4096, 0, 2049, 15]


@pytest.mark.parametrize("make", [
    lambda: W.tiny(),
    lambda: W.llama8b(B=6, ctx_range=(1, 700)),
    lambda: W.paged("ragged", B=len(RAGGED), Hq=16, Hkv=4, D=128, P=16, context_lens=RAGGED,
                    kv="bf16"),
    lambda: W.int8(B=6, ctx_range=(1, 700)),
    lambda: W.paged("ragged-u8", B=len(RAGGED), Hq=16, Hkv=4, D=128, P=32,
                    context_lens=RAGGED, kv="u8", outlier_frac=0.02),
    lambda: W.fp8(B=5, ctx_range=(1, 600)),
    lambda: W.paged("u4d64", B=5, Hq=4, Hkv=2, D=64, P=32, ctx_range=(1, 300), kv="u4",
                    outlier_frac=0.05),
    lambda: W.int4(B=4, ctx_range=(1, 900)),
], ids=["tiny", "llama8b", "ragged", "int8", "ragged-u8", "fp8", "u4-d64", "int4"])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_fused_step_equals_append_then_decode(make, splits):
    w = make()
    k_new, v_new = w.step_rows_by_sequence()
    # reference: separate append, then decode
    pool_a, bt, ctx, q = device_inputs(w, fill_byte=0x5A)
    device_append(pool_a, w, bt)
    want = pa_decode(pool_a, q, bt, ctx, w.scale, num_splits=splits)
    # fused: the prefill rows, then one call
    pool_b, _, _, _ = device_inputs(w, fill_byte=0x5A)
    device_append(pool_b, w, bt, rows="prefill")
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = pa_decode_append(pool_b, q, k_new.to(DEV), v_new.to(DEV), bt, ctx, w.scale,
                           num_splits=splits, d_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(got, want)
    ok, msg = pool_bytes_equal(pool_b, oracle_pool(w, fill_byte=0x5A))
    assert ok, msg
    ref, _ = oracle.paged_attention(oracle_pool(w), bits(w.q), w.block_tables, w.context_lens,
                                    w.scale)
    assert np.abs(got.cpu().numpy().reshape(-1, w.D) - ref).max() <= 2e-3


def test_fused_step_full_size_llama70b():
    """The bench's workload and launch configuration (automatic splits)."""
    w = W.llama70b()
    k_new, v_new = w.step_rows_by_sequence()
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt, rows="prefill")
    got = pa_decode_append(pool, q, k_new.to(DEV), v_new.to(DEV), bt, ctx, w.scale)
    want = pa_decode(pool, q, bt, ctx, w.scale)   # the rows are in place now
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    _, ref, _ = full_size_reference("llama70b")
    err = np.abs(got.cpu().numpy().reshape(ref.shape) - ref).max()
    print(f"fused step llama70b: all rows, max |gpu - oracle| = {err:.3e}")
    assert err <= 2e-3
    # the stored step rows are the inputs, bit for bit
    P = w.P
    for b in (0, w.B // 2, w.B - 1):
        pos = int(w.context_lens[b]) - 1
        page = int(w.block_tables[b, pos // P])
        assert torch.equal(pool.k[page, :, pos % P].cpu(), k_new[b])
        assert torch.equal(pool.v[page, :, pos % P].cpu(), v_new[b])


@pytest.mark.parametrize("kind", ["u4", "u8", "fp8"])
def test_fused_step_with_rows_of_huge_span(kind):
    """The step's own new row spans 8e4 .. 1e30 (INT4 rows of span 8e4 were
    beyond the f16 range of the weights before the weights were normalised):
    stored bit-exact, nothing flagged, and the output within 2e-6 of the span
    of the oracle's Eq. 1."""
    D, Hkv = 128, 2
    for span in (8e4, 1e12, 1e30):
        w = W.paged("bigscale", B=2, Hq=4, Hkv=Hkv, D=D, P=16, context_lens=[3, 21], kv=kind)
        w.step_v[1, 1] = torch.linspace(-span / 2, span / 2, D).to(torch.bfloat16)
        k_new, v_new = w.step_rows_by_sequence()
        pool, bt, ctx, q = device_inputs(w)
        device_append(pool, w, bt, rows="prefill")
        err = torch.zeros(1, dtype=torch.int32, device=DEV)
        got = pa_decode_append(pool, q, k_new.to(DEV), v_new.to(DEV), bt, ctx, w.scale, d_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        ok, msg = pool_bytes_equal(pool, oracle_pool(w))
        assert ok, msg
        ref, _ = oracle.paged_attention(oracle_pool(w), bits(w.q), w.block_tables,
                                        w.context_lens, w.scale)
        g = got.cpu().numpy().reshape(ref.shape)
        assert np.all(np.isfinite(g))
        e = np.abs(g - ref).max()
        print(f"{kind} span {span:.0e}: max |gpu - oracle| = {e:.3e}")
        assert e <= 2e-6 * span + 2e-3


@pytest.mark.parametrize("kv", ["bf16", "u8", "fp8", "u4"])
def test_host_lengths_schedule_the_step_without_changing_it(kv):
    """pa_decode_append with host_context_lens: a ragged batch over several
    waves (64 sequences x 8 KV heads for 444 slots) runs one split, longest
    context first (bf16, INT8 and FP8 with a deeper shared-memory ring). The
    output equals the plain one-split step bit for bit (the same arithmetic
    per CTA, launched in another order from another ring depth) and the
    oracle within 2e-3; host lengths that are wrong (reversed) change only
    the schedule."""
    w = W.llama8b(B=64, ctx_range=(242, 4095), kv=kv,
                  outlier_frac=0.01 if kv != "bf16" else 0.0)
    k_new, v_new = w.step_rows_by_sequence()
    outs = []
    for lens, splits in ((w.context_lens, 0), (w.context_lens[::-1], 0), (None, 1)):
        pool, bt, ctx, q = device_inputs(w)
        device_append(pool, w, bt, rows="prefill")
        outs.append(pa_decode_append(pool, q, k_new.to(DEV), v_new.to(DEV), bt, ctx, w.scale,
                                     num_splits=splits, host_context_lens=lens))
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[2])
    ref, _ = oracle.paged_attention(oracle_pool(w), bits(w.q), w.block_tables, w.context_lens,
                                    w.scale)
    for o in outs[:2]:
        assert np.abs(o.cpu().numpy().reshape(ref.shape) - ref).max() <= 2e-3
