"""Pins for the CPU oracle, checked against the pages and mathematics only.

Nothing here touches the CUDA path. Each test states what fixes the value it
compares against: a number the pages print (tests/golden/), a closed form, a
special case that reduces to a library routine (torch SDPA in float64,
Python's round-half-even), or an invariant of Eq. 1.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_466_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return W.bits(x.to(torch.bfloat16))


def _f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _contiguous_pool(K, V, P):
    """Identity page layout: pages of sequence b are b*npg .. b*npg+npg-1.

    K, V: float tensors [B, Hkv, T, D] with T a multiple of P. Returns the pool
    [B*npg, Hkv, P, D] (bf16 bits) and the identity block table.
    """
    B, Hkv, T, D = K.shape
    npg = T // P
    def to_pool(X):
        X = X.reshape(B, Hkv, npg, P, D).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, P, D)
        return _bf16_bits(X)
    table = np.arange(B * npg, dtype=np.int32).reshape(B, npg)
    return to_pool(K), to_pool(V), table


def _pool(kind, k, v, P, k_sz=None, v_sz=None):
    return oracle.HostPool(kind, P, np.ascontiguousarray(k), np.ascontiguousarray(v),
                           k_sz, v_sz)


def _sdpa_reference(q, K, V, ctx, scale):
    """torch SDPA in float64 with GQA (query head i uses KV head i // G)."""
    B = q.shape[0]
    outs = []
    for b in range(B):
        n = int(ctx[b])
        qb = q[b:b + 1, :, None, :].double()              # [1, Hq, 1, D]
        kb = K[b:b + 1, :, :n, :].double()                # [1, Hkv, n, D]
        vb = V[b:b + 1, :, :n, :].double()
        ob = F.scaled_dot_product_attention(qb, kb, vb, scale=scale, enable_gqa=True)
        outs.append(ob[0, :, 0, :])
    return torch.stack(outs).numpy()


def _rand_case(seed, B=3, Hq=8, Hkv=2, D=64, P=16, T=80):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(B, Hkv, T, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, T, D, generator=g).to(torch.bfloat16)
    return q, K, V


# ---------------------------------------------------------------- Eq. 1 pins
def test_one_token_context_returns_its_value_row():
    """ctx = 1: softmax over one score is exactly 1, so out == v_0 bit for bit."""
    q, K, V = _rand_case(1)
    kp, vp, table = _contiguous_pool(K, V, 16)
    ctx = np.array([1, 1, 1], np.int32)
    out, lse = oracle.paged_attention(_pool("bf16", kp, vp, 16), _bf16_bits(q), table, ctx, 0.125)
    G = 4
    for b in range(3):
        for hq in range(8):
            np.testing.assert_array_equal(out[b * 8 + hq], V[b, hq // G, 0].double().numpy())
            s0 = 0.125 * float(np.dot(_f64(_bf16_bits(q[b, hq])), K[b, hq // G, 0].double().numpy()))
            assert lse[b * 8 + hq] == pytest.approx(s0, abs=1e-12)


def test_uniform_keys_give_mean_of_values():
    """All keys equal: every weight is 1/n, so out = mean of the value rows and
    lse = s + log(n)."""
    q, K, V = _rand_case(2, T=96)
    K[:] = K[:, :, :1, :]
    kp, vp, table = _contiguous_pool(K, V, 16)
    ctx = np.array([96, 50, 7], np.int32)
    out, lse = oracle.paged_attention(_pool("bf16", kp, vp, 16), _bf16_bits(q), table, ctx, 0.2)
    for b in range(3):
        n = int(ctx[b])
        for hq in range(8):
            h = hq // 4
            np.testing.assert_allclose(out[b * 8 + hq], V[b, h, :n].double().mean(0).numpy(),
                                       rtol=0, atol=1e-12)
            s = 0.2 * float(np.dot(q[b, hq].double().numpy(), K[b, h, 0].double().numpy()))
            assert lse[b * 8 + hq] == pytest.approx(s + math.log(n), abs=1e-12)


def test_dominant_key_selects_its_value_row():
    """One score far above the rest: the softmax puts (almost) all weight on it."""
    q, K, V = _rand_case(3, B=1, Hq=2, Hkv=1, T=48)
    q[0, 0] = 0
    q[0, 0, 5] = 1.0
    K[0, 0, 37, 5] = 512.0          # s_37 = 512 * scale = 64 above the others
    kp, vp, table = _contiguous_pool(K, V, 16)
    out, _ = oracle.paged_attention(_pool("bf16", kp, vp, 16), _bf16_bits(q), table,
                                    np.array([48], np.int32), 0.125, pairs=[(0, 0)])
    np.testing.assert_allclose(out[0], V[0, 0, 37].double().numpy(), atol=1e-20)


@pytest.mark.parametrize("seed,Hq,Hkv,D,P", [(4, 8, 2, 64, 16), (5, 4, 4, 128, 32),
                                             (6, 8, 1, 64, 16), (7, 16, 2, 128, 16)])
def test_matches_torch_sdpa_float64(seed, Hq, Hkv, D, P):
    """Identity page layout reduces Eq. 1 to textbook attention: compare with
    torch.nn.functional.scaled_dot_product_attention in float64 (enable_gqa)."""
    q, K, V = _rand_case(seed, B=3, Hq=Hq, Hkv=Hkv, D=D, P=P, T=4 * P)
    kp, vp, table = _contiguous_pool(K, V, P)
    ctx = np.array([4 * P, 3 * P - 5, 1], np.int32)     # full, ragged, single token
    scale = 1.0 / math.sqrt(D)
    out, _ = oracle.paged_attention(_pool("bf16", kp, vp, P), _bf16_bits(q), table, ctx, scale)
    ref = _sdpa_reference(q, K, V, ctx, scale).reshape(-1, D)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_page_permutation_invariance_is_exact():
    """Paging must not change results: moving pages around the pool and
    updating the tables gives the identical fp64 output ("without changing
    model output", PagedAttention Solution)."""
    q, K, V = _rand_case(8, B=4, T=64)
    kp, vp, table = _contiguous_pool(K, V, 16)
    ctx = np.array([64, 33, 17, 2], np.int32)
    base, base_lse = oracle.paged_attention(_pool("bf16", kp, vp, 16), _bf16_bits(q), table,
                                            ctx, 0.125)
    rng = np.random.default_rng(0)
    for _ in range(3):
        n = kp.shape[0]
        extra = 7
        perm = rng.permutation(n + extra)            # new physical id of old page i = perm[i]
        kq = np.full((n + extra,) + kp.shape[1:], 0x7FC0, np.uint16)   # NaN filler
        vq = kq.copy()
        kq[perm[:n]] = kp
        vq[perm[:n]] = vp
        t2 = perm[table].astype(np.int32)
        out, lse = oracle.paged_attention(_pool("bf16", kq, vq, 16), _bf16_bits(q), t2, ctx, 0.125)
        np.testing.assert_array_equal(out, base)
        np.testing.assert_array_equal(lse, base_lse)


def test_slots_beyond_context_are_never_read():
    """Tokens at or past ctx (NaN here) and table entries past ceil(ctx/P)
    (-1 here) do not affect the result."""
    q, K, V = _rand_case(9, B=2, T=64)
    kp, vp, table = _contiguous_pool(K, V, 16)
    ctx = np.array([21, 40], np.int32)
    ref, _ = oracle.paged_attention(_pool("bf16", kp, vp, 16), _bf16_bits(q), table, ctx, 0.125)
    kp2, vp2, t2 = kp.copy(), vp.copy(), table.copy()
    for b in range(2):
        n = int(ctx[b])
        for t in range(n, 64):
            kp2[table[b, t // 16], :, t % 16] = 0x7FC0
            vp2[table[b, t // 16], :, t % 16] = 0x7FC0
        t2[b, -(-n // 16):] = -1
    out, _ = oracle.paged_attention(_pool("bf16", kp2, vp2, 16), _bf16_bits(q), t2, ctx, 0.125)
    np.testing.assert_array_equal(out, ref)


def test_empty_context_gives_zero_and_minus_inf():
    q, K, V = _rand_case(10, B=1, T=16)
    kp, vp, table = _contiguous_pool(K, V, 16)
    out, lse = oracle.paged_attention(_pool("bf16", kp, vp, 16), _bf16_bits(q), table,
                                      np.array([0], np.int32), 0.125)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_bad_table_entry_is_reported():
    q, K, V = _rand_case(11, B=1, T=32)
    kp, vp, table = _contiguous_pool(K, V, 16)
    table[0, 1] = 99
    with pytest.raises(ValueError):
        oracle.paged_attention(_pool("bf16", kp, vp, 16), _bf16_bits(q), table,
                               np.array([20], np.int32), 0.125)


def test_fp8_dequantisation_uses_the_scale():
    """E4M3 codes with s = 1/4: the FP8 pool must give the same fp64 output as
    a bf16 pool holding s * value(code) (exact in bf16: 3 mantissa bits)."""
    g = torch.Generator().manual_seed(32)
    B, Hkv, T, D, P = 2, 2, 48, 64, 16
    q = torch.randn(B, 4, D, generator=g).to(torch.bfloat16)
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    idx = torch.randint(0, len(finite), (2, B, Hkv, T, D), generator=g)
    codes = torch.tensor(finite)[idx]
    table = torch.tensor([oracle.e4m3_value(c) if c not in (0x7F, 0xFF) else 0.0
                          for c in range(256)], dtype=torch.float64)
    Kx, Vx = table[codes[0]] / 4, table[codes[1]] / 4
    assert torch.equal(Kx.to(torch.bfloat16).double(), Kx)
    kp, vp, table_ids = _contiguous_pool(Kx.float(), Vx.float(), P)
    npg = T // P
    def to_pool(C):
        return C.reshape(B, Hkv, npg, P, D).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, P, D) \
            .numpy().astype(np.uint8)
    sz = np.zeros((B * npg, Hkv, P, 2), np.float32)
    sz[..., 0] = 0.25
    ctx = np.array([48, 29], np.int32)
    ref, _ = oracle.paged_attention(_pool("bf16", kp, vp, P), _bf16_bits(q), table_ids, ctx, 0.125)
    out, _ = oracle.paged_attention(_pool("fp8", to_pool(codes[0]), to_pool(codes[1]), P, sz,
                                          sz.copy()), _bf16_bits(q), table_ids, ctx, 0.125)
    np.testing.assert_array_equal(out, ref)


def test_int8_dequantisation_uses_scale_and_zero():
    """Eq. 3 right-hand side: with s = 1/8 and z = -16, s*code + z is an exact
    bf16 value, so the INT8 pool must give the same fp64 output as a bf16 pool
    holding those values. Swapping s and z, or dropping either, fails."""
    g = torch.Generator().manual_seed(12)
    B, Hkv, T, D, P = 2, 2, 48, 64, 16
    q = torch.randn(B, 4, D, generator=g).to(torch.bfloat16)
    codes_k = torch.randint(0, 256, (B, Hkv, T, D), generator=g, dtype=torch.int32)
    codes_v = torch.randint(0, 256, (B, Hkv, T, D), generator=g, dtype=torch.int32)
    Kx = codes_k.double() / 8 - 16
    Vx = codes_v.double() / 8 - 16
    kp, vp, table = _contiguous_pool(Kx.float(), Vx.float(), P)
    assert torch.equal(Kx.to(torch.bfloat16).double(), Kx)    # exact in bf16
    npg = T // P
    def to_pool_u8(C):
        return C.reshape(B, Hkv, npg, P, D).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, P, D) \
            .numpy().astype(np.uint8)
    sz = np.zeros((B * npg, Hkv, P, 2), np.float32)
    sz[..., 0] = 0.125
    sz[..., 1] = -16.0
    ctx = np.array([48, 29], np.int32)
    ref, _ = oracle.paged_attention(_pool("bf16", kp, vp, P), _bf16_bits(q), table, ctx, 0.125)
    out, _ = oracle.paged_attention(_pool("u8", to_pool_u8(codes_k), to_pool_u8(codes_v), P,
                                          sz, sz.copy()), _bf16_bits(q), table, ctx, 0.125)
    np.testing.assert_array_equal(out, ref)


def test_lse_merge_recovers_whole_range():
    """Softmax over a union of disjoint ranges = LSE-weighted merge of the
    per-range results; an empty range (lse = -inf) has no effect."""
    q, K, V = _rand_case(13, B=2, T=96)
    kp, vp, table = _contiguous_pool(K, V, 16)
    ctx = np.array([96, 70], np.int32)
    pool = _pool("bf16", kp, vp, 16)
    qb = _bf16_bits(q)
    whole, whole_lse = oracle.paged_attention(pool, qb, table, ctx, 0.125)
    cuts = [0, 13, 40, 40, 96]          # includes an empty range [40, 40)
    parts, lses = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, l = oracle.paged_attention(pool, qb, table, ctx, 0.125, t_begin=a, t_end=b)
        parts.append(o)
        lses.append(l)
    o = np.stack(parts, 1)
    l = np.stack(lses, 1)
    merged = oracle.lse_merge(o, l)
    np.testing.assert_allclose(merged, whole, rtol=0, atol=1e-12)
    M = l.max(1)
    np.testing.assert_allclose(M + np.log(np.exp(l - M[:, None]).sum(1)), whole_lse,
                               rtol=0, atol=1e-12)
    assert np.all(oracle.lse_merge(np.zeros((3, 2, 4)), np.full((3, 2), -np.inf)) == 0)


def test_scatter_follows_the_block_table_diagram(golden_dir):
    """Logical position -> (physical page, slot) for the page-2 diagram's
    table [42, 7, 89] with 16-token blocks, written out by hand."""
    spec = json.load(open(os.path.join(golden_dir, "block_table_diagram.json")))
    P = spec["page_size"]
    pool = oracle.empty_pool("bf16", spec["pool_pages"], 1, P, 8, fill_byte=0)
    table = np.array([spec["block_table"]], np.int32)
    pos = np.array([c["pos"] for c in spec["cases"]], np.int32)
    marks = (np.arange(len(pos), dtype=np.uint16) + 1)[:, None, None] * np.ones((1, 1, 8), np.uint16)
    oracle.scatter_rows(pool, table, np.zeros(len(pos), np.int32), pos, marks, marks)
    for i, c in enumerate(spec["cases"]):
        assert np.all(pool.k[c["page"], 0, c["slot"]] == i + 1), c
    assert np.count_nonzero(pool.k) == len(pos) * 8


# ------------------------------------------------------ Eq. 5 / Eq. 6 pins
def test_window_covering_everything_is_full_attention():
    """window >= ctx (or window = 0) keeps every token: identical to Eq. 1."""
    q, K, V = _rand_case(20, B=3, T=64)
    kp, vp, table = _contiguous_pool(K, V, 16)
    pool = _pool("bf16", kp, vp, 16)
    ctx = np.array([64, 41, 5], np.int32)
    full, full_lse = oracle.paged_attention(pool, _bf16_bits(q), table, ctx, 0.125)
    for sinks, window in [(0, 0), (0, 64), (3, 100), (4, 60)]:
        out, lse = oracle.paged_attention_window(pool, _bf16_bits(q), table, ctx, 0.125,
                                                 sinks, window)
        np.testing.assert_array_equal(out, full)
        np.testing.assert_array_equal(lse, full_lse)


def test_window_of_one_returns_the_newest_value_row():
    q, K, V = _rand_case(21, B=3, T=48)
    kp, vp, table = _contiguous_pool(K, V, 16)
    ctx = np.array([48, 17, 2], np.int32)
    out, _ = oracle.paged_attention_window(_pool("bf16", kp, vp, 16), _bf16_bits(q), table,
                                           ctx, 0.125, 0, 1)
    for b in range(3):
        for hq in range(8):
            np.testing.assert_array_equal(out[b * 8 + hq], V[b, hq // 4, ctx[b] - 1].double().numpy())


def test_sinks_and_window_equal_attention_over_the_kept_tokens():
    """Eq. 5 as a token set: copy only the kept tokens (first s, last w) into
    a fresh contiguous cache and run plain Eq. 1 on it; the results agree."""
    q, K, V = _rand_case(22, B=3, Hq=8, Hkv=2, T=96)
    kp, vp, table = _contiguous_pool(K, V, 16)
    ctx = np.array([96, 70, 30], np.int32)
    sinks, window = 4, 37
    got, got_lse = oracle.paged_attention_window(_pool("bf16", kp, vp, 16), _bf16_bits(q),
                                                 table, ctx, 0.125, sinks, window)
    for b in range(3):
        n = int(ctx[b])
        keep = [t for t in range(n) if t < sinks or t >= n - window]
        Kk = K[b:b + 1, :, keep, :]
        Vk = V[b:b + 1, :, keep, :]
        T2 = -(-len(keep) // 16) * 16
        Kp = torch.zeros(1, 2, T2, 64, dtype=torch.bfloat16); Kp[:, :, :len(keep)] = Kk
        Vp = torch.zeros(1, 2, T2, 64, dtype=torch.bfloat16); Vp[:, :, :len(keep)] = Vk
        kp2, vp2, t2 = _contiguous_pool(Kp, Vp, 16)
        ref, ref_lse = oracle.paged_attention(_pool("bf16", kp2, vp2, 16), _bf16_bits(q[b:b + 1]),
                                              t2, np.array([len(keep)], np.int32), 0.125)
        np.testing.assert_allclose(got[b * 8:(b + 1) * 8], ref, rtol=0, atol=1e-13)
        np.testing.assert_allclose(got_lse[b * 8:(b + 1) * 8], ref_lse, rtol=0, atol=1e-13)


# ------------------------------------------------------------------ Eq. 3 pins
def _row_bits(vals):
    t = torch.tensor(vals, dtype=torch.float32)
    assert torch.equal(t.to(torch.bfloat16).float(), t), "test values must be exact bf16"
    return _bf16_bits(t)[None, :]


def test_quantiser_rounds_half_to_even_unit_scale():
    """min 0, max 255 -> s = 1, z = 0, so code = round_half_even(x); compare
    with Python's round(), which rounds halves to even."""
    vals = [0.0, 255.0, 0.5, 1.5, 2.5, 3.5, 126.5, 127.5, 0.25, 0.75, 100.0, 64.5]
    codes, sz = oracle.quantize_rows(_row_bits(vals))
    assert sz[0, 0] == 1.0 and sz[0, 1] == 0.0
    assert codes[0].tolist() == [round(v) for v in vals]


def test_quantiser_rounds_half_to_even_half_scale():
    """min -1, max 126.5 -> range 127.5, s = 0.5 exactly, z = -1."""
    vals = [-1.0, 126.5, -0.75, -0.25, 0.25, 0.75, 10.25, 11.75]
    codes, sz = oracle.quantize_rows(_row_bits(vals))
    assert sz[0, 0] == 0.5 and sz[0, 1] == -1.0
    assert codes[0].tolist() == [round((v + 1.0) * 2) for v in vals]


def test_quantiser_constant_row():
    codes, sz = oracle.quantize_rows(_row_bits([3.25] * 16))
    assert sz[0, 0] == 0.0 and sz[0, 1] == 3.25 and np.all(codes == 0)


def test_quantiser_signed_zero_has_one_pattern():
    """A row whose minimum is a zero stores z = +0 whatever the zero's sign,
    and an all-zero row stores s = +0."""
    for vals in ([-0.0, 0.0, 1.0, 2.0], [0.0, -0.0, 1.0, 2.0], [-0.0] * 4, [0.0, -0.0] * 2):
        codes, sz = oracle.quantize_rows(_row_bits(vals))
        assert sz.view(np.uint32)[0, 1] == 0 and sz.view(np.uint32)[0, 0] in (0, np.float32(2 / 255).view(np.uint32))


def test_quantiser_endpoints_and_round_trip_bound():
    """min -> code 0, max -> code 255, and |x - (s*code + z)| <= s/2 up to
    fp32 rounding of the ratio (255 ulp-sized steps at most)."""
    g = torch.Generator().manual_seed(14)
    x = (torch.randn(500, 128, generator=g) * torch.rand(500, 1, generator=g) * 4)
    x[:, 7] += 30 * torch.rand(500, generator=g)        # outliers
    xb = _bf16_bits(x)
    codes, sz = oracle.quantize_rows(xb)
    xf = _f64(xb)
    s = sz[:, 0].astype(np.float64)
    z = sz[:, 1].astype(np.float64)
    assert np.all(z == xf.min(1))
    assert np.all(codes[np.arange(500), xf.argmin(1)] == 0)
    assert np.all(codes[np.arange(500), xf.argmax(1)] == 255)
    rel = (xf.max(1) - xf.min(1)) / 255.0
    assert np.all(np.abs(s - rel) <= rel * 2.0 ** -22)
    err = np.abs(xf - (s[:, None] * codes + z[:, None]))
    assert np.all(err <= s[:, None] * (0.5 + 255 * 2.0 ** -22) + 1e-30)


# ----------------------------------------------------------- INT4 pins
def test_int4_quantiser_half_even_and_nibble_order():
    """min 0, max 15 -> s = 1: codes are Python's round-half-even of x; element
    2i sits in the low nibble of byte i, element 2i + 1 in the high nibble."""
    vals = [0.0, 15.0, 1.0, 2.0, 0.5, 1.5, 2.5, 7.5, 14.5, 3.25, 9.75, 12.0]
    packed, sz = oracle.quantize_rows_int4(_row_bits(vals))
    assert sz[0, 0] == 1.0 and sz[0, 1] == 0.0
    assert packed[0, 0] == 0xF0 and packed[0, 1] == 0x21
    codes = oracle.unpack_int4(packed)[0].tolist()
    assert codes == [round(v) for v in vals]


def test_int4_quantiser_endpoints_constant_row_and_bound():
    g = torch.Generator().manual_seed(40)
    x = torch.randn(400, 64, generator=g) * torch.rand(400, 1, generator=g) * 3
    x[5] = 1.5
    xb = _bf16_bits(x)
    packed, sz = oracle.quantize_rows_int4(xb)
    codes = oracle.unpack_int4(packed)
    xf = _f64(xb)
    assert sz[5, 0] == 0 and sz[5, 1] == 1.5 and np.all(codes[5] == 0)
    rows = np.flatnonzero(sz[:, 0] > 0)
    assert np.all(codes[rows, xf[rows].argmin(1)] == 0)
    assert np.all(codes[rows, xf[rows].argmax(1)] == 15)
    s = sz[:, 0:1].astype(np.float64)
    err = np.abs(xf - (s * codes + sz[:, 1:2]))
    assert np.all(err <= s * (0.5 + 15 * 2.0 ** -22) + 1e-30)


def test_int4_dequantisation_uses_scale_zero_and_nibbles():
    """s = 1, z = -8: s*code + z is exact in bf16, so an INT4 pool must give the
    same fp64 attention as a bf16 pool of those values (a nibble or order
    mix-up, or a swapped s and z, fails)."""
    g = torch.Generator().manual_seed(41)
    B, Hkv, T, D, P = 2, 2, 48, 64, 16
    q = torch.randn(B, 4, D, generator=g).to(torch.bfloat16)
    ck = torch.randint(0, 16, (B, Hkv, T, D), generator=g)
    cv = torch.randint(0, 16, (B, Hkv, T, D), generator=g)
    kp, vp, table = _contiguous_pool((ck - 8).float(), (cv - 8).float(), P)
    npg = T // P
    def to_pool(C):
        C = C.reshape(B, Hkv, npg, P, D).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, P, D)
        C = C.numpy().astype(np.uint8)
        return (C[..., 0::2] | (C[..., 1::2] << 4)).astype(np.uint8)
    sz = np.zeros((B * npg, Hkv, P, 2), np.float32)
    sz[..., 0] = 1.0
    sz[..., 1] = -8.0
    ctx = np.array([48, 29], np.int32)
    ref, _ = oracle.paged_attention(_pool("bf16", kp, vp, P), _bf16_bits(q), table, ctx, 0.125)
    out, _ = oracle.paged_attention(_pool("u4", to_pool(ck), to_pool(cv), P, sz, sz.copy()),
                                    _bf16_bits(q), table, ctx, 0.125)
    np.testing.assert_array_equal(out, ref)


# ------------------------------------------------------- FP8 (E4M3) pins
def test_e4m3_code_table_from_the_format_definition():
    """1 sign, 4 exponent bits (bias 7), 3 mantissa bits; no infinities;
    S.1111.111 is NaN; subnormals have exponent 2^-6 and quantum 2^-9."""
    assert oracle.e4m3_value(0x00) == 0.0 and oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9 and oracle.e4m3_value(0x08) == 2.0 ** -6
    assert oracle.e4m3_value(0x38) == 1.0 and oracle.e4m3_value(0x7E) == 448.0
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(vals, vals[1:]))             # strictly increasing
    for c in range(0x7F):
        assert oracle.e4m3_value(0x80 | c) == -vals[c] or (c == 0)
        assert oracle.e4m3_encode(vals[c]) == c                     # exact values round trip
        if c:
            assert oracle.e4m3_encode(-vals[c]) == 0x80 | c


def test_e4m3_rounding_matches_torch_float8_e4m3fn():
    """Round to nearest, ties to even: agree with torch's float8_e4m3fn cast
    (a library routine) on random values of every magnitude in range."""
    g = torch.Generator().manual_seed(30)
    mag = torch.exp2(torch.rand(200_000, generator=g) * 18 - 11)       # 2^-11 .. 2^7
    x = (mag * torch.sign(torch.randn(200_000, generator=g))).float()
    mids = torch.tensor([(oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2
                         for c in range(0x7E)], dtype=torch.float32)   # exact ties
    x = torch.cat([x, mids, -mids, torch.tensor([448.0, 447.0, 460.0, -460.0])])
    want = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x.tolist()], np.uint8)
    np.testing.assert_array_equal(got, want)


def test_fp8_quantiser_scale_endpoints_and_bound():
    """s = max|x| / 448 per row; the largest element maps to +-448 exactly; a
    zero row stores s = 0; |x - s*E4M3(code)| <= s * half the code spacing."""
    g = torch.Generator().manual_seed(31)
    x = torch.randn(300, 128, generator=g) * torch.rand(300, 1, generator=g) * 5
    x[3] = 0
    xb = _bf16_bits(x)
    codes, sz = oracle.quantize_rows_fp8(xb)
    xf = _f64(xb)
    amax = np.abs(xf).max(1)
    np.testing.assert_array_equal(sz[:, 0], (amax.astype(np.float32) / np.float32(448)))
    assert np.all(sz[:, 1] == 0) and sz[3, 0] == 0 and np.all(codes[3] == 0)
    table = np.array([oracle.e4m3_value(c) for c in range(256)])
    rows = np.arange(300)[amax > 0]
    top = np.abs(xf[rows]).argmax(1)
    assert np.all(np.isin(codes[rows, top], (0x7E, 0xFE)))
    deq = sz[:, :1].astype(np.float64) * table[codes]
    r = np.abs(xf) / np.where(sz[:, :1] > 0, sz[:, :1], 1)
    spacing = np.where(r < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(r, 2.0 ** -6))) - 3))
    assert np.all(np.abs(xf - deq) <= sz[:, :1] * (0.5 * spacing * (1 + 2.0 ** -20)) + 1e-30)


# ---------------------------------------------- Eq. 2 and the memory formula
def test_memory_formula_llama3_70b(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "memory_formula.json")))
    one = oracle.kv_memory_bytes(spec["layers"], spec["kv_heads"], spec["head_dim"],
                                 spec["tokens"], spec["bytes_per_elem"])
    assert one == spec["printed_bytes"]
    assert round(one / 1e9, 2) == spec["printed_gb_rounded"]
    batch = spec["batch"] * one
    assert batch == 85_899_345_920 == 80 * 2 ** 30
    assert batch > 80e9                           # more than an 80 GB A100 holds
    assert abs(batch / 1e9 - spec["printed_batch_gb"]) < 0.25


def test_exercise3_seven_billion_model():
    """Exercise 3 (L=32, H=32, d_k=128, T=4096): fp16 2 GiB, INT8 half, INT4
    a quarter, and GQA with G=4 of 32 heads scales by 4/32 (Eq. 7)."""
    fp16 = oracle.kv_memory_bytes(32, 32, 128, 4096, 2)
    assert fp16 == 2 ** 31
    assert oracle.kv_memory_bytes(32, 32, 128, 4096, 1) == fp16 // 2
    assert oracle.kv_memory_bytes(32, 32, 128, 4096, 0.5) == fp16 // 4
    assert oracle.kv_memory_bytes(32, 4, 128, 4096, 0.5) == fp16 // 32


def test_cache_ratios(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "cache_ratios.json")))
    H, G = spec["gqa"]["H"], spec["gqa"]["G"]
    mha = oracle.kv_memory_bytes(80, H, 128, 1000, 2)
    gqa = oracle.kv_memory_bytes(80, G, 128, 1000, 2)
    assert mha // gqa == spec["gqa"]["printed_reduction"]
    assert mha // oracle.kv_memory_bytes(80, G, 128, 1000, 0.5) == spec["gqa_int4"]["printed_reduction"]
    q = spec["quantisation"]
    assert oracle.kv_memory_bytes(1, 1, 128, 10, 2) / oracle.kv_memory_bytes(1, 1, 128, 10, 1) == q["fp16_to_int8"]
    assert oracle.kv_memory_bytes(1, 1, 128, 10, 2) / oracle.kv_memory_bytes(1, 1, 128, 10, 0.5) == q["fp16_to_int4"]
    w = spec["paging_waste"]
    assert oracle.max_internal_waste_tokens(w["page_size"]) == w["max_waste_tokens"]
    # a request of T tokens leaves ceil(T/P)*P - T <= P-1 slots empty
    for T in range(1, 200):
        assert -(-T // 16) * 16 - T <= w["max_waste_tokens"]
    assert w["static_T"] - 1 > w["max_waste_tokens"]


def test_eq2_closed_forms(golden_dir):
    spec = json.load(open(os.path.join(golden_dir, "cache_ratios.json")))["prefix"]
    N, Ps = spec["N"], spec["P_shared"]
    for T in (2000, 2500, 4096):
        saved = oracle.eq2_paged(N, T) - oracle.eq2_prefix_cached(N, T, Ps)
        assert saved == (N - 1) * Ps
    assert spec["printed_saving_tokens"] == N * Ps     # the page's own rounding
    lengths = [2000 + s for s in (1, 17, 512, 300)]
    assert oracle.eq2_paged_var(lengths) - oracle.eq2_prefix_cached_var(lengths, 2000) == 3 * 2000
    assert oracle.eq2_pages_unshared(lengths, 16) - oracle.eq2_pages_shared(lengths, 2000, 16) \
        == 3 * 125


def test_eq2_shared_prefix_workload():
    """The 128-request shared-prefix workload: storing the 125-page prefix
    once saves exactly 127 * 125 = 15,875 pages (Eq. 2 in page units), and
    its two pools have exactly those sizes."""
    shared, unshared = W.prefix()
    lengths = shared.context_lens.tolist()
    pu = oracle.eq2_pages_unshared(lengths, 16)
    ps = oracle.eq2_pages_shared(lengths, 2000, 16)
    assert pu - ps == 15_875
    assert shared.num_pages == ps and unshared.num_pages == pu
