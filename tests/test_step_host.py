"""pa_decode_step_host: one decode step from a host packet (one H2D copy,
append, decode, one D2H copy) must give exactly what the separate device
calls give, and the oracle's Eq. 1 within tolerance."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_466_b200 import (KVPool, StepPacket, _lib, pa_decode, pa_decode_auto_splits,
                                     pa_decode_num_splits, pa_decode_step_host)
from paged_kv_cache_466_b200 import workloads as W
from paged_kv_cache_466_b200.workloads import bits
from tests.helpers import DEV, device_append, device_inputs, oracle_pool, pool_bytes_equal

TOL = 2e-3


def test_packet_layout_is_packed_in_order_and_256_aligned():
    pool = KVPool(4, 8, 32, 128, "bf16", device="cpu")
    B, Hq, mp, n = 3, 64, 17, 5
    p = StepPacket(pool, B, Hq, mp, n, pin=False)
    sizes = [B * Hq * 128 * 2, n * 8 * 128 * 2, n * 8 * 128 * 2, n * 4, n * 4, B * mp * 4, B * 4]
    assert p.offsets[0] == 0
    for i in range(7):
        assert p.offsets[i] % 256 == 0
        end = p.offsets[i] + sizes[i]
        nxt = p.offsets[i + 1] if i < 6 else p.nbytes
        assert end <= nxt < end + 256
    assert p.nbytes % 256 == 0
    assert p.q.shape == (B, Hq, 128) and p.block_tables.shape == (B, mp)
    # one row per sequence: B rows of K/V, no index sections
    p1 = StepPacket(pool, B, Hq, mp, -1, pin=False)
    assert p1.k_new.shape == (B, 8, 128) and p1.seq_idx.numel() == 0 and p1.pos.numel() == 0
    assert p1.offsets[3] == p1.offsets[4] == p1.offsets[5]
    assert p.k_new.shape == (n, 8, 128) and p.context_lens.shape == (B,)
    # the views alias the packet bytes
    p.context_lens[1] = 0x01020304
    assert bytes(p.host[p.offsets[6] + 4:p.offsets[6] + 8].numpy()) == b"\x04\x03\x02\x01"


def _fill(packet, w, rows=True):
    packet.q.copy_(w.q)
    if rows:
        packet.k_new.copy_(w.step_k)
        packet.v_new.copy_(w.step_v)
        packet.seq_idx.copy_(torch.from_numpy(w.step_seq))
        packet.pos.copy_(torch.from_numpy(w.step_pos))
    packet.block_tables.copy_(torch.from_numpy(w.block_tables))
    packet.context_lens.copy_(torch.from_numpy(w.context_lens))


@pytest.mark.gpu
@pytest.mark.parametrize("make", [
    lambda: W.llama8b(B=6, ctx_range=(1, 700)),
    lambda: W.int8(B=5, ctx_range=(1, 500)),
    lambda: W.paged("u4p32", B=4, Hq=16, Hkv=2, D=64, P=32, ctx_range=(1, 300), kv="u4"),
], ids=["bf16", "int8", "int4-d64"])
@pytest.mark.parametrize("sync", [True, False])
def test_step_host_equals_the_device_calls(make, sync):
    w = make()
    # reference: the prefill rows, then this step's rows and the decode as separate calls
    pool_a, bt, ctx, q = device_inputs(w)
    device_append(pool_a, w, bt)
    want = pa_decode(pool_a, q, bt, ctx, w.scale)
    # the step: same prefill, then the packet carries the step rows and the query
    pool_b, _, _, _ = device_inputs(w)
    device_append(pool_b, w, bt, rows="prefill")
    packet = StepPacket(pool_b, w.B, w.Hq, w.max_pages, len(w.step_seq))
    _fill(packet, w)
    out_host = torch.full((w.B, w.Hq, w.D), float("nan")).pin_memory()
    pa_decode_step_host(pool_b, packet, w.scale, out_host, synchronize=sync)
    if not sync:
        torch.cuda.synchronize()
    assert torch.equal(out_host, want.cpu())
    ok, msg = pool_bytes_equal(pool_b, oracle_pool(w))
    assert ok, msg
    ref, _ = oracle.paged_attention(oracle_pool(w), bits(w.q), w.block_tables, w.context_lens,
                                    w.scale)
    assert np.abs(out_host.numpy().reshape(-1, w.D) - ref).max() <= TOL


@pytest.mark.gpu
def test_step_host_without_new_rows_and_bad_packet_size():
    w = W.tiny()
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt)
    packet = StepPacket(pool, w.B, w.Hq, w.max_pages, 0)
    _fill(packet, w, rows=False)
    out_host = torch.empty((w.B, w.Hq, w.D)).pin_memory()
    pa_decode_step_host(pool, packet, w.scale, out_host)
    assert torch.equal(out_host, pa_decode(pool, q, bt, ctx, w.scale).cpu())
    out_dev = torch.empty((w.B, w.Hq, w.D), device=DEV)
    st = _lib.load().pa_decode_step_host(
        ctypes.byref(pool.c), ctypes.c_void_p(packet.host.data_ptr()),
        ctypes.c_void_p(packet.dev.data_ptr()), packet.nbytes + 256, w.B, w.Hq, w.max_pages, 0,
        w.scale, ctypes.c_void_p(out_dev.data_ptr()), ctypes.c_void_p(out_host.data_ptr()),
        None, 0, 1, None, None, 1)
    assert st == _lib.PA_ERR_INVALID_ARG
    assert b"packet_bytes" in _lib.load().pa_last_error()


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hkv,ctx,P", [(32, 8, 8192, 32), (64, 8, 4095, 16), (4, 2, 64, 16),
                                          (1, 1, 30000, 32), (0, 8, 100, 16)])
def test_auto_splits_is_the_planner_for_a_bf16_d128_pool(B, Hkv, ctx, P):
    pool = KVPool(4, Hkv, P, 128, "bf16", DEV)
    assert pa_decode_auto_splits(B, Hkv, ctx, P) == pa_decode_num_splits(pool, B, -(-ctx // P))


@pytest.mark.gpu
@pytest.mark.parametrize("make", [lambda: W.llama8b(B=6, ctx_range=(1, 700)),
                                  lambda: W.int8(B=5, ctx_range=(1, 500))], ids=["bf16", "int8"])
def test_step_host_one_row_per_sequence_runs_the_fused_step(make):
    from paged_kv_cache_466_b200 import PA_STEP_NEWEST_PER_SEQ
    w = make()
    k_new, v_new = w.step_rows_by_sequence()
    pool_a, bt, ctx, q = device_inputs(w)
    device_append(pool_a, w, bt)
    want = pa_decode(pool_a, q, bt, ctx, w.scale)
    pool_b, _, _, _ = device_inputs(w)
    device_append(pool_b, w, bt, rows="prefill")
    packet = StepPacket(pool_b, w.B, w.Hq, w.max_pages, PA_STEP_NEWEST_PER_SEQ)
    assert packet.k_new.shape == (w.B, w.Hkv, w.D) and packet.seq_idx.numel() == 0
    packet.q.copy_(w.q)
    packet.k_new.copy_(k_new)
    packet.v_new.copy_(v_new)
    packet.block_tables.copy_(torch.from_numpy(w.block_tables))
    packet.context_lens.copy_(torch.from_numpy(w.context_lens))
    out_host = torch.full((w.B, w.Hq, w.D), float("nan")).pin_memory()
    pa_decode_step_host(pool_b, packet, w.scale, out_host)
    assert torch.equal(out_host, want.cpu())
    ok, msg = pool_bytes_equal(pool_b, oracle_pool(w))
    assert ok, msg


@pytest.mark.gpu
@pytest.mark.parametrize("per_seq", [True, False], ids=["fused", "append+decode"])
def test_step_graph_replays_the_step_with_new_packet_contents(per_seq):
    from paged_kv_cache_466_b200 import PA_STEP_NEWEST_PER_SEQ, StepGraph
    w = W.int8(B=5, ctx_range=(1, 500))
    pool, bt, ctx, q = device_inputs(w)
    device_append(pool, w, bt, rows="prefill")
    n = PA_STEP_NEWEST_PER_SEQ if per_seq else len(w.step_seq)
    packet = StepPacket(pool, w.B, w.Hq, w.max_pages, n)
    if per_seq:
        k_new, v_new = w.step_rows_by_sequence()
        packet.k_new.copy_(k_new)
        packet.v_new.copy_(v_new)
    else:
        packet.k_new.copy_(w.step_k)
        packet.v_new.copy_(w.step_v)
        packet.seq_idx.copy_(torch.from_numpy(w.step_seq))
        packet.pos.copy_(torch.from_numpy(w.step_pos))
    packet.block_tables.copy_(torch.from_numpy(w.block_tables))
    packet.context_lens.copy_(torch.from_numpy(w.context_lens))
    out_host = torch.full((w.B, w.Hq, w.D), float("nan")).pin_memory()
    graph = StepGraph(pool, packet, w.scale, out_host)
    try:
        for scale_q in (1.0, -0.5):          # new query each step, same cache
            qq = (w.q.float() * scale_q).to(torch.bfloat16)
            packet.q.copy_(qq)
            got = graph.launch().clone()
            want = pa_decode(pool, qq.to(DEV), bt, ctx, w.scale).cpu()
            assert torch.equal(got, want)
        ok, msg = pool_bytes_equal(pool, oracle_pool(w))
        assert ok, msg
    finally:
        graph.close()
