"""pa_decode on the GPU against the fp64 oracle (Eq. 1 over gathered pages).

Tolerance: max-abs 2e-3 on the fp32 outputs (the bound the task sets for
attention computed from identical bf16 or dequantised inputs). The kernels
are much closer than that (~1e-5: fp32 accumulation, softmax weights kept to
~16 bits), and the tests print the observed error.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_466_b200 import (PA_DERR_BAD_CTX, PA_DERR_BAD_PAGE, pa_decode,
                                     pa_decode_num_splits, pa_decode_workspace_bytes,
                                     pa_splitkv_reduce, pa_validate_tables)
from paged_kv_cache_466_b200 import workloads as W
from paged_kv_cache_466_b200.workloads import bits
import oracle
from tests.helpers import (DEV, device_append, device_inputs, full_size_reference,
                           oracle_decode, oracle_pool)

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _run(w, num_splits=0, fill_byte=0x00):
    pool, bt, ctx, q = device_inputs(w, fill_byte=fill_byte)
    device_append(pool, w, bt)
    out = pa_decode(pool, q, bt, ctx, w.scale, num_splits=num_splits)
    torch.cuda.synchronize()
    return out.cpu().numpy().reshape(-1, w.D), (pool, bt, ctx, q)


def _check(w, got, pairs=None, tol=TOL):
    hp = oracle_pool(w)
    ref, _ = oracle_decode(w, hp, pairs=pairs)
    if pairs is not None:
        got = np.stack([got[b * w.Hq + h] for b, h in pairs])
    err = np.abs(got.astype(np.float64) - ref).max() if ref.size else 0.0
    print(f"{w.name}: max |gpu - oracle| = {err:.3e}")
    assert np.all(np.isfinite(got))
    assert err <= tol
    return err


SMALL = {
    "tiny": lambda: W.tiny(),
    "llama8b-small": lambda: W.llama8b(B=6, ctx_range=(1, 700)),
    "llama70b-small": lambda: W.llama70b(B=2, ctx=1000),
    "int8-small": lambda: W.int8(B=6, ctx_range=(1, 700)),
    "prefix-small": lambda: W.prefix(B=8, prefix_tokens=64, suffix_range=(1, 50))[0],
    "d64-p32-g1": lambda: W.paged("d64p32", B=3, Hq=4, Hkv=4, D=64, P=32, ctx_range=(1, 200)),
    "d64-u8": lambda: W.paged("d64u8", B=4, Hq=8, Hkv=2, D=64, P=16, ctx_range=(1, 300),
                              kv="u8", outlier_frac=0.01),
    "u8-p32-g8": lambda: W.paged("u8p32", B=3, Hq=16, Hkv=2, D=128, P=32,
                                 ctx_range=(1, 400), kv="u8"),
    "g3": lambda: W.paged("g3", B=3, Hq=6, Hkv=2, D=128, P=16, ctx_range=(1, 100)),
    "fp8-small": lambda: W.fp8(B=6, ctx_range=(1, 700)),
    "fp8-d64-p32-g8": lambda: W.paged("fp8b", B=3, Hq=16, Hkv=2, D=64, P=32,
                                      ctx_range=(1, 400), kv="fp8", outlier_frac=0.02),
    "int4-small": lambda: W.int4(B=6, ctx_range=(1, 700)),
    "int4-d64-p32-g8": lambda: W.paged("u4b", B=3, Hq=16, Hkv=2, D=64, P=32,
                                       ctx_range=(1, 400), kv="u4", outlier_frac=0.02),
    "int4-g1": lambda: W.paged("u4g1", B=3, Hq=4, Hkv=4, D=128, P=16, ctx_range=(1, 300),
                               kv="u4"),
}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_decode_small_matches_oracle(name, num_splits):
    w = SMALL[name]()
    got, _ = _run(w, num_splits=num_splits)
    _check(w, got)


def test_one_token_context_is_exact():
    """ctx = 1: the softmax weight is exactly 1 and out equals v_0 bit for bit."""
    w = W.paged("ctx1", B=5, Hq=16, Hkv=2, D=128, P=16, context_lens=[1] * 5)
    for S in (0, 1, 4):
        got, _ = _run(w, num_splits=S)
        v0 = w.step_v.float().numpy()                   # [B, Hkv, D]: the only token
        want = np.repeat(v0, w.G, axis=1).reshape(-1, w.D)
        np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("kind", ["u4", "u8", "fp8"])
@pytest.mark.parametrize("span", [6.0e4, 1.0e6, 1e12, 1e30, 1e-12, 1e-30])
@pytest.mark.parametrize("which", ["v", "kv"])
def test_quantised_rows_of_any_span(kind, span, which):
    """Eq. 3 puts no bound on a row's scale. V rows (and K rows) drawn
    uniformly over a span from 1e-30 to 1e30: the weights' power-of-two
    normalisation keeps every f16 operand in range and at full precision. The
    tolerance is relative to the span (fp32 accumulation, weights carried to
    ~2^-22); with large K spans the softmax is one-hot in both."""
    w = W.paged("bigv", B=3, Hq=8, Hkv=2, D=128, P=16, context_lens=[300, 37, 1], kv=kind)
    g = torch.Generator().manual_seed(5)
    big = lambda t: ((torch.rand(t.shape, generator=g) - 0.5) * span).to(torch.bfloat16)
    w.prefill_v, w.step_v = big(w.prefill_v), big(w.step_v)
    if which == "kv":
        w.prefill_k, w.step_k = big(w.prefill_k), big(w.step_k)
    ref, _ = oracle_decode(w, oracle_pool(w))
    for S in (1, 3):
        got, _ = _run(w, num_splits=S)
        assert np.all(np.isfinite(got))
        err = np.abs(got.astype(np.float64) - ref).max()
        print(f"{kind} {which} span {span:.0e}: max |gpu - oracle| = {err:.3e} "
              f"on outputs up to {np.abs(ref).max():.3e}")
        assert err <= 2e-6 * span


def test_empty_context_gives_zero():
    w = W.paged("ctx0", B=3, Hq=8, Hkv=2, D=128, P=16, context_lens=[5, 7, 9])
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    ctx[1] = 0
    for S in (0, 1, 2):
        out = pa_decode(pool, q, bt, ctx, w.scale, num_splits=S)
        torch.cuda.synchronize()
        assert torch.all(out[1] == 0) and torch.all(torch.isfinite(out))


def test_splits_agree():
    """Any split count gives the same answer up to fp32 merge rounding (1e-5)."""
    w = W.llama8b(B=4, ctx_range=(500, 2000))
    outs = [_run(w, num_splits=S)[0] for S in (1, 0, 2, 4, 8, 32, 128)]
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 1e-5


def test_deterministic_and_page_permutation_invariant():
    """Same inputs -> bitwise identical outputs; moving pages to other physical
    ids (and fixing the tables) changes nothing, bitwise."""
    w = W.llama8b(B=5, ctx_range=(100, 900))
    a, (pool, bt, ctx, q) = _run(w)
    out2 = pa_decode(pool, q, bt, ctx, w.scale).cpu().numpy().reshape(-1, w.D)
    np.testing.assert_array_equal(a, out2)
    rng = np.random.default_rng(1)
    perm = rng.permutation(w.num_pages).astype(np.int32)
    w2 = W.llama8b(B=5, ctx_range=(100, 900))
    w2.block_tables = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1) \
        .astype(np.int32)
    b, _ = _run(w2)
    np.testing.assert_array_equal(a, b)


def test_workspace_reuse_across_calls():
    """The split counters in a workspace are re-armed by every call: one
    zero-filled workspace serves many decodes (different batches, split
    counts) with results identical to fresh workspaces."""
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device=DEV)
    for seed, S in [(0, 8), (1, 3), (2, 8), (3, 16)]:
        w = W.llama8b(B=6, ctx_range=(50, 1500), seed=seed)
        pool, bt, ctx, q = device_inputs(w)
        device_append(pool, w, bt)
        fresh = pa_decode(pool, q, bt, ctx, w.scale, num_splits=S)
        reused = pa_decode(pool, q, bt, ctx, w.scale, num_splits=S, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(fresh, reused)


@pytest.mark.parametrize("kv", ["bf16", "u8", "u4"])
def test_automatic_splits_on_ragged_and_empty_contexts(kv):
    """Automatic splitting on a ragged batch: empty sequences between long
    ones, one-token ones, and one long sequence over many splits compared
    with a fixed split count."""
    ctx = [0, 1, 5000, 17, 0, 3, 16, 32, 4096, 0, 2049, 15]
    w = W.paged("ragged", B=len(ctx), Hq=16, Hkv=4, D=128, P=16, context_lens=ctx, kv=kv)
    got, _ = _run(w, num_splits=0)
    _check(w, got)
    # one long sequence over many splits; the same data through 7 fixed splits
    w1 = W.paged("long", B=1, Hq=8, Hkv=1, D=128, P=32, context_lens=[30000], kv=kv)
    a, (pool, bt, ctx1, q) = _run(w1, num_splits=0)
    b = pa_decode(pool, q, bt, ctx1, w1.scale, num_splits=7).cpu().numpy().reshape(-1, w1.D)
    # different partitions: fp32 merge rounding, and for quantised pools the
    # rescaling points of the online softmax differ too
    assert np.abs(a - b).max() <= 5e-5
    _check(w1, a, pairs=[(0, h) for h in range(w1.Hq)])


def test_automatic_splits_workspace_reuse_and_determinism():
    """Automatic splitting re-arms its counters: one zero-filled workspace
    serves many calls, and results repeat bit for bit."""
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device=DEV)
    for seed in range(3):
        w = W.llama8b(B=9, ctx_range=(1, 3000), seed=seed)
        pool, bt, ctx, q = device_inputs(w)
        device_append(pool, w, bt)
        fresh = pa_decode(pool, q, bt, ctx, w.scale)
        r1 = pa_decode(pool, q, bt, ctx, w.scale, workspace=ws)
        r2 = pa_decode(pool, q, bt, ctx, w.scale, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(fresh, r1) and torch.equal(r1, r2)


def test_shared_prefix_equals_unshared_copy_bitwise():
    shared, unshared = W.prefix(B=16, prefix_tokens=160, suffix_range=(1, 100))
    a, _ = _run(shared)
    b, _ = _run(unshared)
    np.testing.assert_array_equal(a, b)
    _check(shared, a)


def test_bad_tables_are_flagged_not_read():
    """Entries outside the pool and impossible context lengths are skipped and
    reported; the other sequences are unaffected."""
    w = W.llama8b(B=4, ctx_range=(40, 300))
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    good = pa_decode(pool, q, bt, ctx, w.scale).clone()
    bt2 = bt.clone()
    bt2[0, 1] = w.num_pages + 100
    bt2[0, 0] = -7
    ctx2 = ctx.clone()
    ctx2[2] = w.max_pages * w.P + 1
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = pa_decode(pool, q, bt2, ctx2, w.scale, d_err=err)
    torch.cuda.synchronize()
    e = int(err.item())
    assert e & PA_DERR_BAD_PAGE and e & PA_DERR_BAD_CTX
    assert torch.all(torch.isfinite(out))
    assert torch.equal(out[1], good[1]) and torch.equal(out[3], good[3])
    assert torch.all(out[2] == 0)
    err.zero_()
    pa_validate_tables(bt2, ctx2, w.num_pages, w.P, err)
    torch.cuda.synchronize()
    assert int(err.item()) == PA_DERR_BAD_PAGE | PA_DERR_BAD_CTX
    err.zero_()
    pa_validate_tables(bt, ctx, w.num_pages, w.P, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_splitkv_reduce_matches_oracle_merge():
    g = torch.Generator().manual_seed(3)
    B, Hq, S, D = 3, 5, 7, 128
    o = torch.randn(B, Hq, S, D, generator=g)
    lse = torch.randn(B, Hq, S, generator=g) * 4
    lse[0, 0, :3] = -float("inf")           # empty splits
    lse[1, 2, :] = -float("inf")            # every split empty -> 0
    got = pa_splitkv_reduce(o.to(DEV), lse.to(DEV)).cpu().numpy()
    want = oracle.lse_merge(o.double().numpy(), lse.double().numpy())
    assert np.abs(got - want).max() <= 1e-5
    assert np.all(got[1, 2] == 0)


def test_workspace_and_split_planning():
    w = W.llama70b(B=2, ctx=256)
    pool, bt, ctx, q = device_inputs(w)
    for req in (0, 1, 3, 8, 1000):
        S = pa_decode_num_splits(pool, w.B, w.max_pages, req)
        assert 1 <= S <= w.max_pages
        C = -(-w.max_pages // S)
        assert -(-w.max_pages // C) == S
        if req:
            assert S <= max(req, 1)
    assert pa_decode_workspace_bytes(2, 64, 128, 1) == 0
    with pytest.raises(Exception):
        pa_decode(pool, q, bt, ctx, w.scale, num_splits=4,
                  workspace=torch.empty(16, dtype=torch.uint8, device=DEV))


# ------------------------------------------------------------------ full sizes
def _check_all_rows(w, ref, got, tol=TOL):
    got = got.reshape(ref.shape)
    assert np.all(np.isfinite(got))
    err = np.abs(got.astype(np.float64) - ref).max()
    worst = np.unravel_index(np.argmax(np.abs(got - ref)), ref.shape)
    print(f"{w.name}: all {ref.shape[0]} rows, max |gpu - oracle| = {err:.3e} at row {worst[0]}")
    assert err <= tol, (w.name, err, worst)
    return err


@pytest.mark.parametrize("name", ["tiny", "llama8b", "llama70b", "int8", "fp8", "int4"])
def test_full_size_outputs(name):
    """The full workloads, in the launch configuration the benchmark times
    (automatic split count), every (sequence, query head) row against the
    oracle."""
    w, ref, _ = full_size_reference(name)
    got, _ = _run(w)
    _check_all_rows(w, ref, got)


@pytest.mark.parametrize("num_splits", [2, 5, 8])
def test_full_size_llama70b_split_kv(num_splits):
    """The Llama-3-70B-shaped batch (32 x 8192 tokens) with its split-KV path
    forced: every row against the oracle (2e-3), and against the unsplit
    decode of the same pool (1e-5: the log-sum-exp merge is exact up to
    rounding)."""
    w, ref, _ = full_size_reference("llama70b")
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    assert pa_decode_num_splits(pool, w.B, w.max_pages, num_splits) == num_splits
    one = pa_decode(pool, q, bt, ctx, w.scale, num_splits=1)
    got = pa_decode(pool, q, bt, ctx, w.scale, num_splits=num_splits)
    torch.cuda.synchronize()
    got_np = got.cpu().numpy().reshape(-1, w.D)
    _check_all_rows(w, ref, got_np)
    d = (got - one).abs().max().item()
    print(f"llama70b S={num_splits} vs S=1: {d:.3e}")
    assert d <= 1e-5


def test_full_size_prefix_shared_equals_unshared():
    shared, unshared = W.prefix()
    a, _ = _run(shared)
    b, _ = _run(unshared)
    np.testing.assert_array_equal(a, b)
    w, ref, _ = full_size_reference("prefix")
    _check_all_rows(w, ref, a)


def test_one_workspace_serves_calls_of_every_shape_and_entry_point():
    """A workspace zero-filled once serves a sequence of calls whose shapes
    grow and shrink and that mix entry points: the split counters sit in a
    region sized by the workspace alone, which no call writes partials into."""
    from paged_kv_cache_466_b200 import pa_decode_range, pa_decode_window
    ws = torch.zeros(48 << 20, dtype=torch.uint8, device=DEV)
    plan = [(W.llama8b(B=6, ctx_range=(1, 3000), seed=4), "decode", 8),
            (W.int8(B=30, ctx_range=(1, 2000), seed=5), "decode", 3),
            (W.llama8b(B=9, ctx_range=(200, 3000), seed=6), "range", 4),
            (W.llama8b(B=40, ctx_range=(1, 1500), seed=7), "decode", 2),
            (W.llama8b(B=7, ctx_range=(500, 3000), seed=8), "window", 3),
            (W.llama8b(B=64, ctx_range=(1, 900), seed=9), "decode", 5)]
    for w, kind, S in plan:
        pool, bt, ctx, q = device_inputs(w)
        device_append(pool, w, bt)
        if kind == "decode":
            got = pa_decode(pool, q, bt, ctx, w.scale, num_splits=S, workspace=ws)
            want = pa_decode(pool, q, bt, ctx, w.scale, num_splits=S)
        elif kind == "range":
            got = pa_decode_range(pool, q, bt, ctx, w.scale, 64, 2500, num_splits=S,
                                  workspace=ws)[0]
            want = pa_decode_range(pool, q, bt, ctx, w.scale, 64, 2500, num_splits=S)[0]
        else:
            got = pa_decode_window(pool, q, bt, ctx, w.scale, 4, 1000, num_splits=S,
                                   workspace=ws)
            want = pa_decode_window(pool, q, bt, ctx, w.scale, 4, 1000, num_splits=S)
        torch.cuda.synchronize()
        assert torch.equal(got, want), (w.name, kind, S)
