"""pa_kv_append on the GPU against the oracle's scatter and Eq. 3 quantiser:
the whole pool must match byte for byte, untouched slots included."""
import numpy as np
import pytest
import torch

from paged_kv_cache_466_b200 import (PA_DERR_BAD_PAGE, PA_DERR_BAD_POS, PA_DERR_BAD_SEQ,
                                     KVPool, pa_kv_append)
from paged_kv_cache_466_b200 import workloads as W
from tests.helpers import DEV, device_append, device_inputs, oracle_pool, pool_bytes_equal

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("make", [
    lambda: W.tiny(),
    lambda: W.llama8b(B=6, ctx_range=(1, 700)),
    lambda: W.paged("p32d64", B=5, Hq=8, Hkv=4, D=64, P=32, ctx_range=(1, 300)),
    lambda: W.int8(B=6, ctx_range=(1, 700)),
    lambda: W.paged("u8d64", B=5, Hq=4, Hkv=2, D=64, P=16, ctx_range=(1, 300), kv="u8",
                    outlier_frac=0.02),
    lambda: W.paged("u8p32", B=3, Hq=16, Hkv=2, D=128, P=32, ctx_range=(1, 200), kv="u8"),
    lambda: W.fp8(B=6, ctx_range=(1, 700)),
    lambda: W.paged("fp8d64", B=5, Hq=4, Hkv=2, D=64, P=32, ctx_range=(1, 300), kv="fp8",
                    outlier_frac=0.05),
    lambda: W.int4(B=6, ctx_range=(1, 700)),
    lambda: W.paged("u4d64", B=5, Hq=4, Hkv=2, D=64, P=32, ctx_range=(1, 300), kv="u4",
                    outlier_frac=0.05),
], ids=["tiny", "llama8b-small", "p32-d64", "int8-small", "int8-d64", "int8-p32", "fp8-small",
        "fp8-d64-p32", "int4-small", "int4-d64-p32"])
def test_append_matches_oracle_scatter_bit_exact(make):
    w = make()
    pool, bt, _, _ = device_inputs(w, fill_byte=0xA5)
    device_append(pool, w, bt)
    torch.cuda.synchronize()
    ok, msg = pool_bytes_equal(pool, oracle_pool(w, fill_byte=0xA5))
    assert ok, msg


def test_append_int8_full_pool_bit_exact():
    """All 9,798 pages of the INT8 workload (Llama-3-8B shapes, 1 % outliers):
    every code and every fp32 scale/zero equals the oracle's."""
    w = W.int8()
    pool, bt, _, _ = device_inputs(w, fill_byte=0x00)
    device_append(pool, w, bt)
    torch.cuda.synchronize()
    ok, msg = pool_bytes_equal(pool, oracle_pool(w, fill_byte=0x00))
    assert ok, msg


def test_append_fp8_full_pool_bit_exact():
    """All pages of the FP8 workload: every E4M3 code and fp32 scale equals the
    oracle's (round to nearest even, saturating, per-row absmax scale)."""
    w = W.fp8()
    pool, bt, _, _ = device_inputs(w, fill_byte=0x00)
    device_append(pool, w, bt)
    torch.cuda.synchronize()
    ok, msg = pool_bytes_equal(pool, oracle_pool(w, fill_byte=0x00))
    assert ok, msg


@pytest.mark.parametrize("kind", ["u8", "fp8", "u4"])
@pytest.mark.parametrize("D", [128, 64])
def test_append_quantiser_edge_rows_all_formats(kind, D):
    Hkv = 2
    rows = []
    rows.append(np.full(D, 3.25, np.float32))
    r = np.zeros(D, np.float32); r[::2] = -0.0; r[5] = 2.0; rows.append(r)
    r = np.arange(D, dtype=np.float32) + 0.5; r[0] = 0.0; r[1] = 255.0; rows.append(r)
    r = np.linspace(-3e4, 3e4, D).astype(np.float32); rows.append(r)
    r = np.linspace(-1e-30, 1e-30, D).astype(np.float32); rows.append(r)
    r = np.zeros(D, np.float32); rows.append(r)
    x = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    n = x.shape[0] // Hkv
    k = x[:n * Hkv].reshape(n, Hkv, D)
    w = W.paged("edge", B=1, Hq=2, Hkv=Hkv, D=D, P=16, context_lens=[n], kv=kind)
    w.prefill_k, w.prefill_v = k[:-1].contiguous(), k.flip(0)[:-1].contiguous()
    w.step_k, w.step_v = k[-1:].contiguous(), k.flip(0)[-1:].contiguous()
    pool, bt, _, _ = device_inputs(w)
    device_append(pool, w, bt)
    torch.cuda.synchronize()
    ok, msg = pool_bytes_equal(pool, oracle_pool(w))
    assert ok, msg


def test_append_int4_full_pool_bit_exact():
    """All pages of the INT4 workload: every packed code pair and fp32
    scale/zero equals the oracle's (Eq. 3 with 16 levels)."""
    w = W.int4()
    pool, bt, _, _ = device_inputs(w, fill_byte=0x00)
    device_append(pool, w, bt)
    torch.cuda.synchronize()
    ok, msg = pool_bytes_equal(pool, oracle_pool(w, fill_byte=0x00))
    assert ok, msg


def test_append_quantiser_edge_rows():
    """Constant rows (s = 0), rows with both signed zeros, exact half-way
    ties, huge and tiny magnitudes."""
    D, Hkv = 128, 2
    rows = []
    rows.append(np.full(D, 3.25, np.float32))
    r = np.zeros(D, np.float32); r[::2] = -0.0; r[5] = 2.0; rows.append(r)
    r = np.arange(D, dtype=np.float32) + 0.5; r[0] = 0.0; r[1] = 255.0; rows.append(r)
    r = np.linspace(-3e4, 3e4, D).astype(np.float32); rows.append(r)
    r = np.linspace(-1e-30, 1e-30, D).astype(np.float32); rows.append(r)
    r = np.full(D, -0.0, np.float32); rows.append(r)
    x = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)          # [6, D]
    n = x.shape[0] // Hkv
    k = x[:n * Hkv].reshape(n, Hkv, D)
    w = W.paged("edge", B=1, Hq=2, Hkv=Hkv, D=D, P=16, context_lens=[n], kv="u8")
    w.prefill_k = k[:-1].contiguous()
    w.prefill_v = k.flip(0)[:-1].contiguous()
    w.step_k = k[-1:].contiguous()
    w.step_v = k.flip(0)[-1:].contiguous()
    pool, bt, _, _ = device_inputs(w)
    device_append(pool, w, bt)
    torch.cuda.synchronize()
    ok, msg = pool_bytes_equal(pool, oracle_pool(w))
    assert ok, msg


def test_append_skips_bad_rows_and_flags_them():
    """Rows naming a sequence, position or page outside the tables are skipped
    (nothing written) and reported through the error word."""
    w = W.tiny()
    pool, bt, _, _ = device_inputs(w, fill_byte=0x11)
    before = [t.clone() for t in pool.tensors()]
    Hkv, D = w.Hkv, w.D
    k = torch.randn(4, Hkv, D).to(torch.bfloat16).to(DEV)
    bt_bad = bt.clone()
    bt_bad[1, 0] = w.num_pages + 5                       # page outside the pool
    seq = torch.tensor([-1, 4, 0, 1], dtype=torch.int32, device=DEV)
    pos = torch.tensor([0, 0, 10_000, 3], dtype=torch.int32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pa_kv_append(pool, k, k, seq, pos, bt_bad, d_err=err)
    torch.cuda.synchronize()
    e = int(err.item())
    assert e & PA_DERR_BAD_SEQ and e & PA_DERR_BAD_POS and e & PA_DERR_BAD_PAGE
    for a, b in zip(before, pool.tensors()):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


def test_append_empty_is_noop():
    w = W.tiny()
    pool, bt, _, _ = device_inputs(w, fill_byte=0x22)
    e = torch.empty(0, w.Hkv, w.D, dtype=torch.bfloat16, device=DEV)
    i = torch.empty(0, dtype=torch.int32, device=DEV)
    pa_kv_append(pool, e, e, i, i, bt)
    torch.cuda.synchronize()
    assert torch.all(pool.k.view(torch.uint8) == 0x22)


@pytest.mark.parametrize("kind", ["u4", "u8", "fp8"])
@pytest.mark.parametrize("span", [8e4, 1.2e6, 1e30, 1e-30])
def test_append_stores_rows_of_any_scale(kind, span):
    """Rows with very large and very small spans are stored bit-exact with the
    oracle's quantiser, and the error word stays clear (no row scale is out of
    range for the decode)."""
    D, Hkv = 128, 2
    x = torch.linspace(-span / 2, span / 2, D).to(torch.bfloat16)
    k = torch.zeros(3, Hkv, D, dtype=torch.bfloat16)
    k[1, 1] = x
    w = W.paged("bigscale", B=1, Hq=2, Hkv=Hkv, D=D, P=16, context_lens=[3], kv=kind)
    w.prefill_k, w.prefill_v = k[:2].contiguous(), k[:2].flip(1).contiguous()
    w.step_k, w.step_v = k[2:].contiguous(), k[2:].contiguous()
    pool, bt, _, _ = device_inputs(w)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    device_append(pool, w, bt, d_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ok, msg = pool_bytes_equal(pool, oracle_pool(w))
    assert ok, msg
