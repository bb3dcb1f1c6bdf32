"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest

from paged_kv_cache_466_b200 import _lib
from paged_kv_cache_466_b200._lib import (PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED,
                                          PA_ERR_WORKSPACE, PA_OK, pa_kv_pool_t)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_466_b200 import build
    build.build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert {"pa_kv_append", "pa_decode", "pa_splitkv_reduce"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(_lib.SIGNATURES) == declared


def test_version_and_status_strings(lib):
    assert lib.pa_abi_version() == 2
    for s in range(7):
        assert lib.pa_status_str(s) and lib.pa_status_str(s) != b"unknown status"
    assert lib.pa_status_str(99) == b"unknown status"


def _pool(**kw):
    p = dict(num_pages=8, page_size=16, num_kv_heads=2, head_dim=128, dtype=0,
             k_pool=0x1000, v_pool=0x2000, k_sz=None, v_sz=None)
    p.update(kw)
    return pa_kv_pool_t(**p)


def _decode(lib, pool, B=2, Hq=4, max_pages=4, ws=None, ws_bytes=0, splits=0, q=0x3000,
            out=0x4000, scale=0.1):
    return lib.pa_decode(ctypes.byref(pool) if pool is not None else None, q, B, Hq, 0x5000,
                         max_pages, 0x6000, scale, out, ws, ws_bytes, splits, None, None)


def test_decode_rejects_bad_arguments(lib):
    assert _decode(lib, None) == PA_ERR_INVALID_ARG
    assert _decode(lib, _pool(head_dim=96)) == PA_ERR_UNSUPPORTED
    assert _decode(lib, _pool(page_size=8)) == PA_ERR_UNSUPPORTED
    assert _decode(lib, _pool(dtype=7)) == PA_ERR_UNSUPPORTED
    assert _decode(lib, _pool(dtype=1)) == PA_ERR_INVALID_ARG          # no k_sz / v_sz
    assert _decode(lib, _pool(k_pool=0x1001)) == PA_ERR_INVALID_ARG    # misaligned
    assert _decode(lib, _pool(), Hq=5) == PA_ERR_INVALID_ARG           # 5 % 2 != 0
    assert _decode(lib, _pool(), Hq=18) == PA_ERR_UNSUPPORTED          # group of 9
    assert _decode(lib, _pool(), q=None) == PA_ERR_INVALID_ARG
    assert _decode(lib, _pool(), out=0x4004) == PA_ERR_INVALID_ARG
    assert _decode(lib, _pool(), scale=float("nan")) == PA_ERR_INVALID_ARG
    assert _decode(lib, _pool(), splits=-1) == PA_ERR_INVALID_ARG
    assert b"multiple" in lib.pa_last_error() or lib.pa_last_error()
    # more than one split needs a workspace
    assert _decode(lib, _pool(), splits=2) == PA_ERR_WORKSPACE
    need = lib.pa_decode_workspace_bytes(2, 4, 128, 2)
    assert _decode(lib, _pool(), splits=2, ws=0x10010, ws_bytes=need) == PA_ERR_WORKSPACE
    assert _decode(lib, _pool(), splits=2, ws=0x10000, ws_bytes=need - 1) == PA_ERR_WORKSPACE
    assert _decode(lib, _pool(), B=0) == PA_OK                          # nothing to do


def test_append_and_reduce_reject_bad_arguments(lib):
    pool = _pool()
    args = [ctypes.byref(pool), 0x1000, 0x2000, 0x3000, 0x4000, 4, 0x5000, 2, 4, None, None]
    bad = list(args); bad[1] = None
    assert lib.pa_kv_append(*bad) == PA_ERR_INVALID_ARG
    bad = list(args); bad[5] = -1
    assert lib.pa_kv_append(*bad) == PA_ERR_INVALID_ARG
    bad = list(args); bad[2] = 0x2002
    assert lib.pa_kv_append(*bad) == PA_ERR_INVALID_ARG
    bad = list(args); bad[5] = 0
    assert lib.pa_kv_append(*bad) == PA_OK                              # empty append
    assert lib.pa_splitkv_reduce(0x1000, 0x2000, 2, 4, 0, 128, 0x3000, None) == PA_ERR_INVALID_ARG
    assert lib.pa_splitkv_reduce(0x1000, 0x2000, 2, 4, 2, 130, 0x3000, None) == PA_ERR_INVALID_ARG
    assert lib.pa_splitkv_reduce(None, 0x2000, 2, 4, 2, 128, 0x3000, None) == PA_ERR_INVALID_ARG
    assert lib.pa_splitkv_reduce(0x1000, 0x2000, 0, 4, 2, 128, 0x3000, None) == PA_OK
    assert lib.pa_validate_tables(0x1000, 2, 4, 0x2000, 8, 16, None, None) == PA_ERR_INVALID_ARG


def test_split_planning_and_workspace_size(lib):
    pool = _pool(page_size=32)
    for B, mp, req in [(32, 256, 0), (1, 1, 0), (64, 256, 5), (3, 4000, 1), (2, 100, 1000)]:
        S = lib.pa_decode_num_splits(ctypes.byref(pool), B, mp, req)
        assert 1 <= S <= min(mp, 256)
        C = -(-mp // S)
        assert -(-mp // C) == S                       # no empty split by construction
        assert C <= 2048
    assert lib.pa_decode_num_splits(ctypes.byref(pool), 4, 4000, 1) == 2   # 2048-entry cap
    assert lib.pa_decode_num_splits(ctypes.byref(pool), 4, 0, 0) <= 0
    assert lib.pa_decode_workspace_bytes(32, 64, 128, 1) == 0
    for B, Hq, D, S in [(32, 64, 128, 8), (1, 8, 64, 2), (4096, 64, 128, 2), (7, 12, 64, 3)]:
        ws = lib.pa_decode_workspace_bytes(B, Hq, D, S)
        rest = -(-B * Hq * S * D * 4 // 256) * 256 + -(-B * Hq * S * 4 // 256) * 256
        c = B * Hq * 4
        assert ws % 256 == 0
        # the counter region is [0, 256 * (size // 32768)); the partials follow it,
        # for the returned size and for every larger one
        for size in (ws, ws + 1, ws + 255, ws + 32768 * 3 - ws % 32768, 2 * ws):
            region = 256 * (size // 32768)
            assert region >= c and size - region >= rest, (B, Hq, D, S, size)
        # about 1/128 over the parts, the counter region at least 256 bytes (32 KB)
        assert ws <= max(rest * 128 / 127, 128 * c) + 33280


def test_device_error_words_map_to_statuses(lib):
    from paged_kv_cache_466_b200._lib import (PA_DERR_BAD_CTX, PA_DERR_BAD_PAGE,
                                              PA_DERR_BAD_POS, PA_DERR_BAD_SEQ,
                                              PA_DERR_TIMEOUT, PA_ERR_BAD_TABLE,
                                              PA_ERR_TIMEOUT)
    assert lib.pa_derr_status(0) == PA_OK
    for bit in (PA_DERR_BAD_PAGE, PA_DERR_BAD_CTX, PA_DERR_BAD_SEQ, PA_DERR_BAD_POS):
        assert lib.pa_derr_status(bit) == PA_ERR_BAD_TABLE
        assert lib.pa_derr_status(bit | 16) == PA_ERR_BAD_TABLE
        assert lib.pa_derr_status(bit | PA_DERR_TIMEOUT) == PA_ERR_TIMEOUT
    assert lib.pa_derr_status(PA_DERR_TIMEOUT) == PA_ERR_TIMEOUT
    for bit in (16, 64):      # bits no kernel sets
        assert lib.pa_derr_status(bit) == PA_ERR_INVALID_ARG


def test_auto_splits_and_step_host_reject_bad_arguments(lib):
    assert lib.pa_decode_auto_splits(-1, 8, 100, 16) <= 0
    assert lib.pa_decode_auto_splits(4, 0, 100, 16) <= 0
    assert lib.pa_decode_auto_splits(4, 8, -5, 16) <= 0
    pool = _pool()
    n = lib.pa_step_packet_layout(ctypes.byref(pool), 2, 4, 4, 3, None)
    assert n > 0 and n % 256 == 0
    assert lib.pa_step_packet_layout(ctypes.byref(pool), 2, 4, 0, 3, None) == 0

    def step(nbytes=n, dev=0x20000, host=0x30000):
        return lib.pa_decode_step_host(ctypes.byref(pool), host, dev, nbytes, 2, 4, 4, 3, 0.1,
                                       0x40000, 0x50000, None, 0, 1, None, None, 1)
    assert step(nbytes=n + 256) == PA_ERR_INVALID_ARG
    assert step(dev=0x20010) == PA_ERR_INVALID_ARG
    assert step(host=None) == PA_ERR_INVALID_ARG


def test_selftest_wait_timeout_rejects_bad_limits(lib):
    assert lib.pa_selftest_wait_timeout(0, 0x1000, None) == PA_ERR_INVALID_ARG
    assert lib.pa_selftest_wait_timeout(2_000_000, 0x1000, None) == PA_ERR_INVALID_ARG
    assert lib.pa_selftest_wait_timeout(100, None, None) == PA_ERR_INVALID_ARG


def test_step_graph_rejects_bad_arguments(lib):
    h = ctypes.c_void_p(1234)
    st = lib.pa_step_graph_create(None, None, None, 0, 1, 1, 1, 1, 0.1, None, None, None, 0, 0,
                                  None, ctypes.byref(h))
    assert st == PA_ERR_INVALID_ARG and h.value is None
    assert lib.pa_step_graph_create(ctypes.byref(_pool()), None, None, 0, 0, 1, 1, 1, 0.1, None,
                                    None, None, 0, 0, None, ctypes.byref(h)) == PA_ERR_INVALID_ARG
    assert lib.pa_step_graph_launch(None, None, 1) == PA_ERR_INVALID_ARG
    lib.pa_step_graph_destroy(None)


def test_split_plan_rules_on_a_b200(lib):
    """The planner's two regimes with the B200's 148 SMs and 3 decode CTAs per
    SM (R = 444 slots). One wave when the units fit: the fewest splits that
    give ~1.7 CTAs per SM (252), never a second wave. Otherwise the wave model
    (the split counts measured best on the Llama-3-shaped batches)."""
    plan = lambda units, pages, P, req=0, sms=148, cps=3: lib.pa_decode_plan_splits(
        units, pages, P, sms, cps, req)
    assert plan(32 * 8, 256, 32) == 1          # Llama-3-70B B=32 x 8192: one CTA per unit
    assert plan(16 * 8, 256, 32) == 2
    assert plan(8 * 8, 256, 32) == 4
    assert plan(250, 256, 32) == 1             # 2 splits would spill past 444 slots
    assert plan(200, 256, 32) == 2
    assert plan(32 * 8, 65, 32) == 1           # the 2048-token window + sink pages
    assert plan(64 * 8, 256, 16) == 4          # ragged Llama-3-8B-shaped batch (wave model)
    assert plan(64 * 8, 256, 32) == 6          # B=64 x 8192 (wave model)
    assert plan(0, 10, 16) == 1
    assert plan(8, 4, 16) == 4                 # no more splits than pages
    assert plan(64, 256, 32, req=5) == 5
    assert plan(4, 4000, 32, req=1) == 2       # a split stages at most 2048 table entries
    assert plan(100, 256, 32, sms=132, cps=2) == 2   # another GPU: R = 264, target 225
    assert plan(-1, 4, 16) <= 0 and plan(4, 0, 16) <= 0 and plan(4, 4, 16, sms=0) <= 0


def _prefix_shape(B, prefix, suffix_max, G=4, Hkv=8, D=128, P=16):
    """(units, tiles, estimated suffix bytes) of a cascade batch, as the
    library derives them: 128-row query tiles x KV heads, 64-token prefix
    tiles, half of the table's suffix capacity in bf16 K and V rows."""
    units = -(-(B * G) // 128) * Hkv
    tiles = -(-prefix // 64)
    capacity = -(-suffix_max // P) * P
    return units, tiles, B * Hkv * 2 * (2 * D) * capacity / 2


def test_prefix_plan_rules_on_a_b200(lib):
    """The cascade's prefix split rule with the B200's 148 SMs and 3 decode
    CTAs per SM. Each shape's answer is the split count measured fastest for
    it (cascade step with the prefix pass beside the suffix decode, split
    counts 1..32 swept): long suffixes leave the SMs to the decode, long
    prefixes spread over all of them."""
    plan = lambda B, pre, sfx, sms=148, cps=3: lib.pa_prefix_plan_splits(
        *_prefix_shape(B, pre, sfx)[:2], sms, cps, _prefix_shape(B, pre, sfx)[2])
    splits = lambda B, pre, sfx: -(-_prefix_shape(B, pre, sfx)[1] // plan(B, pre, sfx))
    assert plan(128, 2000, 512) == 11 and splits(128, 2000, 512) == 3    # 96 CTAs (bench)
    assert splits(32, 2000, 512) == 16                                  # 128 CTAs
    assert splits(64, 4000, 256) == 9                                   # 144 CTAs
    assert splits(128, 8000, 64) == 8                                   # 256 CTAs
    assert splits(256, 1024, 1024) == 1                                 # 64 CTAs
    # no suffix: the fastest prefix pass; equal estimates keep fewer CTAs
    # (8 splits = 256 CTAs, 12.8 us, ties 16 splits in two waves)
    assert lib.pa_prefix_plan_splits(32, 32, 148, 3, 0.0) == 4
    assert lib.pa_prefix_plan_splits(0, 4, 148, 3, 0.0) <= 0
    assert lib.pa_prefix_plan_splits(4, 0, 148, 3, 0.0) <= 0
    assert lib.pa_prefix_plan_splits(4, 4, 0, 3, 0.0) <= 0
    assert lib.pa_prefix_plan_splits(4, 4, 148, 0, 0.0) <= 0
    assert lib.pa_prefix_plan_splits(4, 4, 148, 3, -1.0) <= 0


def test_prefix_plan_invariants_for_any_shape(lib):
    """Any shape gets a valid tile count per split (1..tiles, at most 256
    splits), and a larger suffix never gives the prefix pass more CTAs."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=300, deadline=None)
    @given(units=st.integers(1, 512), tiles=st.integers(1, 2000), sms=st.integers(1, 200),
           cps=st.integers(1, 8), mb=st.floats(0, 4000), more=st.floats(1, 10))
    def check(units, tiles, sms, cps, mb, more):
        tp = lib.pa_prefix_plan_splits(units, tiles, sms, cps, mb * 1e6)
        assert 1 <= tp <= tiles and -(-tiles // tp) <= 256
        tp2 = lib.pa_prefix_plan_splits(units, tiles, sms, cps, mb * 1e6 * more)
        assert -(-tiles // tp2) <= -(-tiles // tp)

    check()


def _plan_lens(lib, lens, hkv=8, max_pages=256, P=16, sms=148, cps=3):
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    order = np.zeros(max(len(lens), 1), dtype=np.uint16)
    S = lib.pa_decode_plan_lens(lens.ctypes.data, len(lens), hkv, max_pages, P, sms, cps,
                                order.ctypes.data)
    return S, order[:len(lens)]


def test_length_aware_plan_on_a_b200(lib):
    """pa_decode_plan_lens with the B200's 148 SMs: a ragged batch that needs
    several waves (64 x 8 = 512 units for 444 slots, contexts 242..4095 as in
    the Llama-3-8B-shaped bench batch) runs one split, longest first; a
    uniform one, a batch that fits one wave, and tables longer than one split
    can stage keep the planner's count."""
    rng = np.random.default_rng(0)
    ragged = rng.integers(242, 4096, 64)
    S, order = _plan_lens(lib, ragged)
    assert S == 1
    assert sorted(order.tolist()) == list(range(64))
    assert all(ragged[order[i]] >= ragged[order[i + 1]] for i in range(63))
    uniform = np.full(64, 4095)
    assert _plan_lens(lib, uniform)[0] == lib.pa_decode_plan_splits(512, 256, 16, 148, 3, 0) == 4
    assert _plan_lens(lib, ragged[:32])[0] == lib.pa_decode_plan_splits(256, 256, 16, 148, 3, 0)
    assert _plan_lens(lib, ragged, max_pages=4096)[0] == \
        lib.pa_decode_plan_splits(512, 4096, 16, 148, 3, 0)
    # four CTAs per SM are planned as three (the planner's calibration)
    assert _plan_lens(lib, ragged, cps=4)[0] == 1
    # ties keep index order; values are clamped to the table
    S, order = _plan_lens(lib, [5, 7, 7, 1 << 30, -3])
    assert order.tolist() == [3, 1, 2, 0, 4]
    bad = np.zeros(4, dtype=np.int32)
    o = np.zeros(4, dtype=np.uint16)
    assert lib.pa_decode_plan_lens(None, 4, 8, 256, 16, 148, 3, o.ctypes.data) <= 0
    assert lib.pa_decode_plan_lens(bad.ctypes.data, 0, 8, 256, 16, 148, 3, o.ctypes.data) <= 0
    big = np.zeros(257, dtype=np.int32)
    ob = np.zeros(257, dtype=np.uint16)
    assert lib.pa_decode_plan_lens(big.ctypes.data, 257, 8, 256, 16, 148, 3, ob.ctypes.data) <= 0


def test_length_aware_plan_invariants(lib):
    """Any lengths: the order is a permutation sorted longest first (ties by
    index), and the count is 1 or the planner's automatic count."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=300, deadline=None)
    @given(lens=st.lists(st.integers(-10, 100000), min_size=1, max_size=256),
           hkv=st.integers(1, 16), pages=st.integers(1, 3000), sms=st.integers(1, 200),
           cps=st.integers(1, 6))
    def check(lens, hkv, pages, sms, cps):
        S, order = _plan_lens(lib, lens, hkv=hkv, max_pages=pages, sms=sms, cps=cps)
        assert S in (1, lib.pa_decode_plan_splits(len(lens) * hkv, pages, 16, sms, min(cps, 3), 0))
        assert sorted(order.tolist()) == list(range(len(lens)))
        clamp = [min(max(x, 0), pages * 16) for x in lens]
        for i in range(len(lens) - 1):
            a, b = order[i], order[i + 1]
            assert clamp[a] > clamp[b] or (clamp[a] == clamp[b] and a < b)

    check()


def test_header_compiles_as_c99_and_host_calls_work(lib, tmp_path):
    """The header is plain C: a C99 program built against it alone links the
    library and runs every entry point that needs no GPU."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = str(tmp_path / "abi_host_calls")
    src = os.path.join(ROOT, "tests", "c", "abi_host_calls.c")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        src, "-o", exe, "-L", libdir, "-lpagedattn", "-Wl,-rpath," + libdir],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "ok" in r.stdout


def test_split_plan_invariants_for_any_shape(lib):
    """For random shapes and device sizes the plan is a valid partition: S in
    [1, min(max_pages, 256)], no empty split, at most 2048 pages per split, an
    honoured request where the limits allow it, and a single wave whenever
    the units fit in the resident slots."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=400, deadline=None)
    @given(units=st.integers(0, 70000), pages=st.integers(1, 20000), P=st.sampled_from([16, 32]),
           sms=st.integers(1, 200), cps=st.integers(1, 8), req=st.integers(0, 300))
    def check(units, pages, P, sms, cps, req):
        S = lib.pa_decode_plan_splits(units, pages, P, sms, cps, req)
        assert 1 <= S <= min(pages, 256)
        C = -(-pages // S)
        assert -(-pages // C) == S and C <= 2048
        lo = -(-pages // 2048)
        if req > 0 and lo <= req <= min(pages, 256) and -(-pages // -(-pages // req)) == req:
            assert S == req
        if req == 0 and 0 < units < sms * cps and lo == 1:
            assert units * S <= sms * cps          # never a second wave

    check()


def test_workspace_sizes_fit_every_larger_buffer(lib):
    """The advertised workspace size, and every larger size, holds the split
    counters in the size-only region and the partials after it."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=300, deadline=None)
    @given(B=st.integers(1, 4096), Hq=st.sampled_from([4, 8, 16, 32, 64, 128]),
           D=st.sampled_from([64, 128]), S=st.integers(2, 256), extra=st.integers(0, 1 << 22))
    def check(B, Hq, D, S, extra):
        ws = lib.pa_decode_workspace_bytes(B, Hq, D, S)
        rest = -(-B * Hq * S * D * 4 // 256) * 256 + -(-B * Hq * S * 4 // 256) * 256
        size = ws + extra
        region = 256 * (size // 32768)
        assert region >= B * Hq * 4 and size - region >= rest

    check()
