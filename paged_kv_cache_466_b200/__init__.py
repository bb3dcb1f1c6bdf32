"""pagedattn for B200: paged KV-cache decode attention behind a C ABI.

The Python layer only marshals arguments: it takes torch tensors, passes their
device pointers and torch's current CUDA stream to ``libpagedattn.so``, and
raises on a non-OK status. Every step of the computation runs in the library's
CUDA kernels; there is no Python or CPU fallback.

Entry points (same names as the C ABI, see include/pagedattn.h):

* ``pa_kv_append``       — write new tokens' K/V into their page slots
                           (quantising for an INT8 pool, Eq. 3)
* ``pa_decode``          — Eq. 1 decode attention over the paged cache
* ``pa_splitkv_reduce``  — log-sum-exp merge of split-KV partials
* ``pa_validate_tables`` — device-side page-table check
* ``pa_decode_num_splits`` / ``pa_decode_workspace_bytes`` — planning helpers
* ``pa_decode_shared_prefix`` — cascade decode for requests sharing a prefix:
                           the prefix as one tensor-core pass for all requests,
                           then the paged decode of each request's own tokens
* ``pa_decode_window``   — decode over attention sinks + the last w tokens
                           (StreamingLLM / sliding window); evicted pages unread
* ``pa_decode_noalloc``  — pa_decode without a caller workspace, for callers
                           that cannot allocate device memory (the scratch is
                           a fixed-size array owned by the library)

``KVPool`` owns the page pool tensors; ``pages`` holds the host-side page
allocator and cache-size formulas.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np
import torch

from . import _lib
from ._lib import (PA_DERR_BAD_CTX, PA_DERR_BAD_PAGE, PA_DERR_BAD_POS, PA_DERR_BAD_SEQ,
                   PA_STEP_NEWEST_PER_SEQ,
                   PA_DERR_TIMEOUT,
                   PA_KV_BF16, PA_KV_FP8_PER_TOKEN, PA_KV_U4_PER_TOKEN, PA_KV_U8_PER_TOKEN,
                   PagedAttnError, pa_kv_pool_t)

__all__ = ["KVPool", "pa_kv_append", "pa_decode", "pa_decode_append", "pa_decode_noalloc", "pa_splitkv_reduce",
           "pa_decode_shared_prefix", "pa_decode_shared_prefix_workspace_bytes",
           "pa_decode_window", "pa_decode_window_workspace_bytes",
           "pa_decode_range", "pa_decode_range_workspace_bytes", "pa_merge_partials",
           "pa_validate_tables", "StepPacket", "pa_decode_step_host", "StepGraph", "pa_derr_status",
           "pa_decode_auto_splits", "pa_selftest_wait_timeout", "PA_DERR_TIMEOUT",
           "PA_STEP_NEWEST_PER_SEQ",
           "pa_decode_num_splits", "pa_decode_workspace_bytes", "PagedAttnError",
           "PA_KV_BF16", "PA_KV_U8_PER_TOKEN", "PA_KV_FP8_PER_TOKEN", "PA_KV_U4_PER_TOKEN",
           "PA_DERR_BAD_PAGE",
           "PA_DERR_BAD_CTX",
           "PA_DERR_BAD_SEQ", "PA_DERR_BAD_POS",
           "load_library", "pa_decode_num_splits_lens"]


def load_library() -> ctypes.CDLL:
    return _lib.load()


def _ptr(t: Optional[torch.Tensor]):
    # ctypes converts a plain int for a c_void_p parameter
    return None if t is None else t.data_ptr()


try:  # the raw handle without building a Stream object (a few microseconds per call)
    _raw_stream = torch._C._cuda_getCurrentRawStream
except AttributeError:  # pragma: no cover
    _raw_stream = None


def _stream(stream=None):
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None:
        return _raw_stream(torch._C._cuda_getDevice())
    return torch.cuda.current_stream().cuda_stream


def _need(t: torch.Tensor, name: str, dtype, device=None):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


class KVPool:
    """The physical page pool: K and V as [num_pages, Hkv, P, D] tensors:
    ``dtype`` "bf16", "u8" (INT8 codes, Eq. 3), "fp8" (E4M3 codes) or "u4"
    (INT4 codes, two per byte: [num_pages, Hkv, P, D/2]); the quantised ones
    with fp32 [num_pages, Hkv, P, 2] (scale, zero) per row."""

    def __init__(self, num_pages: int, num_kv_heads: int, page_size: int, head_dim: int,
                 dtype: str = "bf16", device="cuda", fill_byte: Optional[int] = None):
        self.num_pages, self.num_kv_heads = num_pages, num_kv_heads
        self.page_size, self.head_dim = page_size, head_dim
        self.kind = dtype
        shape = (num_pages, num_kv_heads, page_size, head_dim // 2 if dtype == "u4" else head_dim)
        tdt = {"bf16": torch.bfloat16, "u8": torch.uint8, "fp8": torch.uint8,
               "u4": torch.uint8}[dtype]
        self.k = torch.empty(shape, dtype=tdt, device=device)
        self.v = torch.empty(shape, dtype=tdt, device=device)
        self.k_sz = self.v_sz = None
        if dtype in ("u8", "fp8", "u4"):
            self.k_sz = torch.empty(shape[:3] + (2,), dtype=torch.float32, device=device)
            self.v_sz = torch.empty(shape[:3] + (2,), dtype=torch.float32, device=device)
        if fill_byte is not None:
            for t in self.tensors():
                t.view(torch.uint8).fill_(fill_byte)
        self._c = pa_kv_pool_t(num_pages, page_size, num_kv_heads, head_dim,
                               {"bf16": PA_KV_BF16, "u8": PA_KV_U8_PER_TOKEN,
                                "fp8": PA_KV_FP8_PER_TOKEN, "u4": PA_KV_U4_PER_TOKEN}[dtype],
                               self.k.data_ptr(), self.v.data_ptr(),
                               None if self.k_sz is None else self.k_sz.data_ptr(),
                               None if self.v_sz is None else self.v_sz.data_ptr())

    def tensors(self):
        return [t for t in (self.k, self.v, self.k_sz, self.v_sz) if t is not None]

    @property
    def c(self) -> pa_kv_pool_t:
        return self._c

    @property
    def device(self):
        return self.k.device


def pa_derr_status(derr: int) -> int:
    """The PA_* status a device error word (read back to the host) stands for."""
    return int(_lib.load().pa_derr_status(int(derr)))


def pa_selftest_wait_timeout(limit_us: int, d_err: torch.Tensor, stream=None) -> None:
    """Run the bounded-wait failure path once: a wait that can never complete
    gives up after ``limit_us`` and sets PA_DERR_TIMEOUT in ``d_err``."""
    _need(d_err, "d_err", torch.int32)
    _lib.check(_lib.load().pa_selftest_wait_timeout(int(limit_us), _ptr(d_err), _stream(stream)),
               "pa_selftest_wait_timeout")


def pa_decode_auto_splits(num_seqs: int, num_kv_heads: int, max_ctx: int, page_size: int) -> int:
    """Split count pa_decode picks automatically for a bf16, head_dim-128 pool of
    this shape and a batch whose longest context is ``max_ctx`` tokens."""
    s = _lib.load().pa_decode_auto_splits(num_seqs, num_kv_heads, max_ctx, page_size)
    if s <= 0:
        raise ValueError("pa_decode_auto_splits: invalid arguments")
    return s


def pa_decode_num_splits(pool: KVPool, num_seqs: int, max_pages: int, requested: int = 0) -> int:
    s = _lib.load().pa_decode_num_splits(ctypes.byref(pool.c), num_seqs, max_pages, requested)
    if s <= 0:
        raise ValueError("pa_decode_num_splits: invalid arguments")
    return s


def pa_decode_num_splits_lens(pool: KVPool, num_seqs: int, max_pages: int, host_context_lens,
                              requested: int = 0) -> int:
    """The split count pa_decode_append with host_context_lens uses."""
    hl = np.ascontiguousarray(np.asarray(host_context_lens, dtype=np.int32))
    return int(_lib.load().pa_decode_num_splits_lens(ctypes.byref(pool.c), num_seqs, max_pages,
                                                     hl.ctypes.data, requested))


def pa_decode_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int,
                              num_splits: int) -> int:
    return int(_lib.load().pa_decode_workspace_bytes(num_seqs, num_q_heads, head_dim, num_splits))


def pa_kv_append(pool: KVPool, k_new: torch.Tensor, v_new: torch.Tensor, seq_idx: torch.Tensor,
                 pos: torch.Tensor, block_tables: torch.Tensor,
                 d_err: Optional[torch.Tensor] = None, stream=None) -> None:
    """Write rows k_new/v_new [N, Hkv, D] (bf16) of token (seq_idx[i], pos[i])."""
    dev = pool.device
    _need(k_new, "k_new", torch.bfloat16, dev)
    _need(v_new, "v_new", torch.bfloat16, dev)
    _need(seq_idx, "seq_idx", torch.int32, dev)
    _need(pos, "pos", torch.int32, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    n = seq_idx.numel()
    if k_new.shape != (n, pool.num_kv_heads, pool.head_dim) or v_new.shape != k_new.shape \
            or pos.numel() != n:
        raise ValueError("pa_kv_append: shape mismatch")
    st = _lib.load().pa_kv_append(ctypes.byref(pool.c), _ptr(k_new), _ptr(v_new), _ptr(seq_idx),
                                  _ptr(pos), n, _ptr(block_tables), block_tables.shape[0],
                                  block_tables.shape[1], _ptr(d_err), _stream(stream))
    _lib.check(st, "pa_kv_append")


def pa_decode(pool: KVPool, q: torch.Tensor, block_tables: torch.Tensor,
              context_lens: torch.Tensor, scale: float, out: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
              d_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Eq. 1 decode: q [B, Hq, D] bf16 -> out [B, Hq, D] fp32.

    ``workspace`` (uint8, >= pa_decode_workspace_bytes, zero-filled before its
    first use) is allocated zero-filled with torch when not given.
    """
    dev = pool.device
    _need(q, "q", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    B, Hq, D = q.shape
    if D != pool.head_dim or block_tables.shape[0] != B or context_lens.numel() != B:
        raise ValueError("pa_decode: shape mismatch")
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev)
    max_pages = block_tables.shape[1]
    if workspace is None:
        S = pa_decode_num_splits(pool, B, max_pages, num_splits)
        need = pa_decode_workspace_bytes(B, Hq, D, S)
        if need > 0:
            workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.load().pa_decode(ctypes.byref(pool.c), _ptr(q), B, Hq, _ptr(block_tables),
                               max_pages, _ptr(context_lens), float(scale), _ptr(out),
                               _ptr(workspace), ws_bytes, num_splits, _ptr(d_err),
                               _stream(stream))
    _lib.check(st, "pa_decode")
    return out



def pa_decode_append(pool: KVPool, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                     block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                     out: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
                     d_err: Optional[torch.Tensor] = None, stream=None,
                     host_context_lens=None) -> torch.Tensor:
    """One decode step in one launch: store k_new / v_new [B, Hkv, D] bf16 at
    position context_lens[b] - 1 of each sequence (as pa_kv_append would),
    then Eq. 1 over tokens 0 .. context_lens[b] - 1 (as pa_decode).
    host_context_lens (optional, int32 numpy array or CPU tensor of the same
    values) lets the library schedule the launch from the real lengths
    (pa_decode_append_lens); the result does not depend on it."""
    dev = pool.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_new, "k_new", torch.bfloat16, dev)
    _need(v_new, "v_new", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    B, Hq, D = q.shape
    if D != pool.head_dim or block_tables.shape[0] != B or context_lens.numel() != B \
            or tuple(k_new.shape) != (B, pool.num_kv_heads, D) or k_new.shape != v_new.shape:
        raise ValueError("pa_decode_append: shape mismatch")
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev)
    max_pages = block_tables.shape[1]
    if workspace is None:
        need = pa_decode_workspace_bytes(B, Hq, D,
                                         pa_decode_num_splits(pool, B, max_pages, num_splits))
        if need > 0:
            workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if host_context_lens is not None:
        hl = host_context_lens
        if not (isinstance(hl, np.ndarray) and hl.dtype == np.int32 and hl.flags.c_contiguous):
            hl = np.ascontiguousarray(np.asarray(hl, dtype=np.int32))
        if hl.shape != (B,):
            raise ValueError("pa_decode_append: host_context_lens must hold one length per sequence")
        st = _lib.load().pa_decode_append_lens(
            ctypes.byref(pool.c), _ptr(q), _ptr(k_new), _ptr(v_new), B, Hq, _ptr(block_tables),
            max_pages, _ptr(context_lens), hl.ctypes.data, float(scale), _ptr(out),
            _ptr(workspace), ws_bytes, num_splits, _ptr(d_err), _stream(stream))
        _lib.check(st, "pa_decode_append_lens")
        return out
    st = _lib.load().pa_decode_append(ctypes.byref(pool.c), _ptr(q), _ptr(k_new), _ptr(v_new), B,
                                      Hq, _ptr(block_tables), max_pages, _ptr(context_lens),
                                      float(scale), _ptr(out), _ptr(workspace), ws_bytes,
                                      num_splits, _ptr(d_err), _stream(stream))
    _lib.check(st, "pa_decode_append")
    return out


def pa_decode_shared_prefix_workspace_bytes(pool: KVPool, num_seqs: int, num_q_heads: int,
                                            max_pages: int, prefix_len: int,
                                            num_splits: int = 0) -> int:
    return int(_lib.load().pa_decode_shared_prefix_workspace_bytes(
        ctypes.byref(pool.c), num_seqs, num_q_heads, max_pages, prefix_len, num_splits))


def pa_decode_shared_prefix(pool: KVPool, q: torch.Tensor, prefix_pages: torch.Tensor,
                            prefix_len: int, block_tables: torch.Tensor,
                            context_lens: torch.Tensor, scale: float,
                            out: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
                            d_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Cascade decode: every request's first ``prefix_len`` tokens are the
    shared pages ``prefix_pages``; result equals pa_decode on full tables."""
    dev = pool.device
    _need(q, "q", torch.bfloat16, dev)
    _need(prefix_pages, "prefix_pages", torch.int32, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    B, Hq, D = q.shape
    if D != pool.head_dim or block_tables.shape[0] != B or context_lens.numel() != B:
        raise ValueError("pa_decode_shared_prefix: shape mismatch")
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev)
    max_pages = block_tables.shape[1]
    if workspace is None:
        need = pa_decode_shared_prefix_workspace_bytes(pool, B, Hq, max_pages, prefix_len,
                                                       num_splits)
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.load().pa_decode_shared_prefix(
        ctypes.byref(pool.c), _ptr(q), B, Hq, _ptr(prefix_pages), int(prefix_len),
        _ptr(block_tables), max_pages, _ptr(context_lens), float(scale), _ptr(out),
        _ptr(workspace), ws_bytes, num_splits, _ptr(d_err), _stream(stream))
    _lib.check(st, "pa_decode_shared_prefix")
    return out


def pa_decode_window_workspace_bytes(pool: KVPool, num_seqs: int, num_q_heads: int,
                                     max_pages: int, sinks: int, window: int,
                                     num_splits: int = 0) -> int:
    return int(_lib.load().pa_decode_window_workspace_bytes(
        ctypes.byref(pool.c), num_seqs, num_q_heads, max_pages, sinks, window, num_splits))


def pa_decode_window(pool: KVPool, q: torch.Tensor, block_tables: torch.Tensor,
                     context_lens: torch.Tensor, scale: float, sinks: int, window: int,
                     out: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
                     d_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode over the first ``sinks`` and the last ``window`` tokens of each
    sequence (StreamingLLM); ``window == 0`` keeps every token."""
    dev = pool.device
    _need(q, "q", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    B, Hq, D = q.shape
    if D != pool.head_dim or block_tables.shape[0] != B or context_lens.numel() != B:
        raise ValueError("pa_decode_window: shape mismatch")
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev)
    max_pages = block_tables.shape[1]
    if workspace is None:
        need = (pa_decode_window_workspace_bytes(pool, B, Hq, max_pages, sinks, window,
                                                 num_splits) if window > 0 else
                pa_decode_workspace_bytes(B, Hq, D,
                                          pa_decode_num_splits(pool, B, max_pages, num_splits)))
        if need > 0:
            workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.load().pa_decode_window(
        ctypes.byref(pool.c), _ptr(q), B, Hq, _ptr(block_tables), max_pages, _ptr(context_lens),
        int(sinks), int(window), float(scale), _ptr(out), _ptr(workspace), ws_bytes,
        num_splits, _ptr(d_err), _stream(stream))
    _lib.check(st, "pa_decode_window")
    return out


class StepPacket:
    """The host and device buffers of one ``pa_decode_step_host`` step.

    ``host`` is one page-locked byte buffer laid out by ``pa_step_packet_layout``;
    fill its views (``q``, ``k_new``, ``v_new``, ``seq_idx``, ``pos``,
    ``block_tables``, ``context_lens``) in place and the whole step's input
    crosses to the device in one copy. ``dev`` is the device copy the kernels
    read from."""

    def __init__(self, pool: KVPool, num_seqs: int, num_q_heads: int, max_pages: int,
                 num_new: int, pin: bool = True):
        # num_new == PA_STEP_NEWEST_PER_SEQ: one row per sequence (its newest
        # token), k_new / v_new are [B, Hkv, D] and the step fuses the cache
        # write into the decode
        off = (ctypes.c_size_t * 7)()
        n = int(_lib.load().pa_step_packet_layout(ctypes.byref(pool.c), num_seqs, num_q_heads,
                                                  max_pages, num_new, off))
        if n == 0:
            raise ValueError("StepPacket: invalid shape")
        self.nbytes = n
        self.offsets = [int(o) for o in off]
        self.shape = (num_seqs, num_q_heads, max_pages, num_new)
        host = torch.zeros(n, dtype=torch.uint8)
        self.host = host.pin_memory() if pin else host
        self.dev = (torch.empty(n, dtype=torch.uint8, device=pool.device)
                    if pool.device.type == "cuda" else None)
        B, Hq, D, Hkv = num_seqs, num_q_heads, pool.head_dim, pool.num_kv_heads

        def view(i, dtype, shape):
            count = 1
            for e in shape:
                count *= e
            nb = count * torch.empty((), dtype=dtype).element_size()
            return self.host[self.offsets[i]:self.offsets[i] + nb].view(dtype).view(shape)

        self.q = view(0, torch.bfloat16, (B, Hq, D))
        per_seq = num_new == _lib.PA_STEP_NEWEST_PER_SEQ
        rows = B if per_seq else num_new
        self.k_new = view(1, torch.bfloat16, (rows, Hkv, D))
        self.v_new = view(2, torch.bfloat16, (rows, Hkv, D))
        self.seq_idx = view(3, torch.int32, (0 if per_seq else num_new,))
        self.pos = view(4, torch.int32, (0 if per_seq else num_new,))
        self.block_tables = view(5, torch.int32, (B, max_pages))
        self.context_lens = view(6, torch.int32, (B,))


def pa_decode_step_host(pool: KVPool, packet: StepPacket, scale: float, out_host: torch.Tensor,
                        out_dev: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
                        d_err: Optional[torch.Tensor] = None, stream=None,
                        synchronize: bool = True) -> torch.Tensor:
    """One decode step from host memory: the packet's inputs go to the device
    in one copy, the new rows are appended, Eq. 1 is decoded and the output is
    copied into ``out_host`` (fp32 [B, Hq, D], pinned for an asynchronous copy);
    with ``synchronize`` the call returns once ``out_host`` holds the result."""
    B, Hq, max_pages, num_new = packet.shape
    D = pool.head_dim
    dev = pool.device
    if packet.dev is None:
        raise ValueError("pa_decode_step_host: the packet has no device buffer")
    if out_host.dtype != torch.float32 or out_host.device.type != "cpu" \
            or not out_host.is_contiguous() or tuple(out_host.shape) != (B, Hq, D):
        raise ValueError("pa_decode_step_host: out_host must be a contiguous host fp32 [B, Hq, D]")
    if out_dev is None:
        out_dev = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    _need(out_dev, "out_dev", torch.float32, dev)
    if workspace is None:
        need = pa_decode_workspace_bytes(B, Hq, D,
                                         pa_decode_num_splits(pool, B, max_pages, num_splits))
        if need > 0:
            workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.load().pa_decode_step_host(
        ctypes.byref(pool.c), ctypes.c_void_p(packet.host.data_ptr()), _ptr(packet.dev),
        packet.nbytes, B, Hq, max_pages, num_new, float(scale), _ptr(out_dev),
        ctypes.c_void_p(out_host.data_ptr()), _ptr(workspace), ws_bytes, num_splits,
        _ptr(d_err), _stream(stream), 1 if synchronize else 0)
    _lib.check(st, "pa_decode_step_host")
    return out_host


class StepGraph:
    """A ``pa_decode_step_host`` step captured once into a CUDA graph: each
    ``launch`` copies the packet's current contents to the device, runs the
    step and copies the output into ``out_host`` with one graph launch. Refill
    the packet's views between launches; every buffer is fixed at creation."""

    def __init__(self, pool: KVPool, packet: StepPacket, scale: float, out_host: torch.Tensor,
                 out_dev: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
                 d_err: Optional[torch.Tensor] = None):
        B, Hq, max_pages, num_new = packet.shape
        D = pool.head_dim
        dev = pool.device
        if packet.dev is None or not packet.host.is_pinned():
            raise ValueError("StepGraph: the packet needs a page-locked host buffer and a "
                             "device copy")
        if out_host.dtype != torch.float32 or not out_host.is_pinned() \
                or not out_host.is_contiguous() or tuple(out_host.shape) != (B, Hq, D):
            raise ValueError("StepGraph: out_host must be a page-locked contiguous fp32 "
                             "[B, Hq, D]")
        if out_dev is None:
            out_dev = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
        _need(out_dev, "out_dev", torch.float32, dev)
        if workspace is None:
            need = pa_decode_workspace_bytes(B, Hq, D,
                                             pa_decode_num_splits(pool, B, max_pages, num_splits))
            if need > 0:
                workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        # keep every buffer the graph points at alive as long as the graph
        self._keep = (pool, packet, out_host, out_dev, workspace, d_err)
        self.out_host = out_host
        handle = ctypes.c_void_p()
        st = _lib.load().pa_step_graph_create(
            ctypes.byref(pool.c), ctypes.c_void_p(packet.host.data_ptr()), _ptr(packet.dev),
            packet.nbytes, B, Hq, max_pages, num_new, float(scale), _ptr(out_dev),
            ctypes.c_void_p(out_host.data_ptr()), _ptr(workspace), ws_bytes, num_splits,
            _ptr(d_err), ctypes.byref(handle))
        _lib.check(st, "pa_step_graph_create")
        self._handle = handle

    def launch(self, stream=None, synchronize: bool = True) -> torch.Tensor:
        if self._handle is None:
            raise ValueError("StepGraph: already closed")
        _lib.check(_lib.load().pa_step_graph_launch(self._handle, _stream(stream),
                                                    1 if synchronize else 0),
                   "pa_step_graph_launch")
        return self.out_host

    def close(self) -> None:
        if getattr(self, "_handle", None) is not None:
            torch.cuda.synchronize(self._keep[3].device)
            _lib.load().pa_step_graph_destroy(self._handle)
            self._handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def pa_decode_noalloc(pool: KVPool, q: torch.Tensor, block_tables: torch.Tensor,
                      context_lens: torch.Tensor, scale: float, out: torch.Tensor,
                      num_splits: int = 0, d_err: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """pa_decode for callers that cannot allocate: the split-KV scratch is the
    library's own fixed-size device array, so ``out`` must be given and nothing
    is allocated here either. Calls that overlap on the GPU share that array
    and must be ordered by the caller."""
    dev = pool.device
    _need(q, "q", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    _need(out, "out", torch.float32, dev)
    B, Hq, D = q.shape
    if D != pool.head_dim or block_tables.shape[0] != B or context_lens.numel() != B \
            or tuple(out.shape) != (B, Hq, D):
        raise ValueError("pa_decode_noalloc: shape mismatch")
    st = _lib.load().pa_decode_noalloc(ctypes.byref(pool.c), _ptr(q), B, Hq, _ptr(block_tables),
                                       block_tables.shape[1], _ptr(context_lens), float(scale),
                                       _ptr(out), num_splits, _ptr(d_err), _stream(stream))
    _lib.check(st, "pa_decode_noalloc")
    return out


def pa_splitkv_reduce(o_part: torch.Tensor, lse: torch.Tensor,
                      out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Merge partials o_part [B, Hq, S, D] with lse [B, Hq, S] -> [B, Hq, D]."""
    _need(o_part, "o_part", torch.float32)
    _need(lse, "lse", torch.float32, o_part.device)
    B, Hq, S, D = o_part.shape
    if lse.shape != (B, Hq, S):
        raise ValueError("pa_splitkv_reduce: shape mismatch")
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=o_part.device)
    _need(out, "out", torch.float32, o_part.device)
    st = _lib.load().pa_splitkv_reduce(_ptr(o_part), _ptr(lse), B, Hq, S, D, _ptr(out),
                                       _stream(stream))
    _lib.check(st, "pa_splitkv_reduce")
    return out


def pa_decode_range_workspace_bytes(pool: KVPool, num_seqs: int, num_q_heads: int,
                                    max_pages: int, tok_begin: int, tok_end: int,
                                    num_splits: int = 0) -> int:
    return int(_lib.load().pa_decode_range_workspace_bytes(
        ctypes.byref(pool.c), num_seqs, num_q_heads, max_pages, tok_begin, tok_end, num_splits))


def pa_decode_range(pool: KVPool, q: torch.Tensor, block_tables: torch.Tensor,
                    context_lens: torch.Tensor, scale: float, tok_begin: int, tok_end: int,
                    o_out: Optional[torch.Tensor] = None, lse_out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, num_splits: int = 0,
                    d_err: Optional[torch.Tensor] = None, stream=None):
    """Attention over tokens [tok_begin, min(ctx, tok_end)) of every sequence:
    returns (o [B, Hq, D] normalised over the range, lse [B, Hq] natural log)."""
    dev = pool.device
    _need(q, "q", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    B, Hq, D = q.shape
    if D != pool.head_dim or block_tables.shape[0] != B or context_lens.numel() != B:
        raise ValueError("pa_decode_range: shape mismatch")
    if o_out is None:
        o_out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    if lse_out is None:
        lse_out = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    _need(o_out, "o_out", torch.float32, dev)
    _need(lse_out, "lse_out", torch.float32, dev)
    if tuple(o_out.shape) != (B, Hq, D) or tuple(lse_out.shape) != (B, Hq):
        raise ValueError("pa_decode_range: o_out must be [B, Hq, D] and lse_out [B, Hq]")
    max_pages = block_tables.shape[1]
    if workspace is None:
        need = pa_decode_range_workspace_bytes(pool, B, Hq, max_pages, tok_begin, tok_end,
                                               num_splits)
        if need > 0:
            workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.load().pa_decode_range(
        ctypes.byref(pool.c), _ptr(q), B, Hq, _ptr(block_tables), max_pages, _ptr(context_lens),
        int(tok_begin), int(tok_end), float(scale), _ptr(o_out), _ptr(lse_out), _ptr(workspace),
        ws_bytes, num_splits, _ptr(d_err), _stream(stream))
    _lib.check(st, "pa_decode_range")
    return o_out, lse_out


def pa_merge_partials(o_parts: torch.Tensor, lse_parts: torch.Tensor,
                      out: Optional[torch.Tensor] = None,
                      lse_out: Optional[torch.Tensor] = None, stream=None):
    """Merge part-major partials o_parts [n, ..., D], lse_parts [n, ...] ->
    (out [..., D], lse [...]) (log-sum-exp weights, in part order). Each part
    must be contiguous; the parts themselves may sit at any stride (e.g.
    views into one all-gathered buffer)."""
    for t, name in ((o_parts, "o_parts"), (lse_parts, "lse_parts")):
        if t.dtype != torch.float32:
            raise TypeError(f"{name} must be torch.float32, got {t.dtype}")
        if t.dim() < 2 or not t[0].is_contiguous() or t.stride(0) < t[0].numel():
            raise ValueError(f"{name}: every part must be contiguous and the parts disjoint")
    if lse_parts.device != o_parts.device:
        raise ValueError("lse_parts must be on the device of o_parts")
    n, D = o_parts.shape[0], o_parts.shape[-1]
    rows = lse_parts[0].numel()
    if lse_parts.shape[0] != n or o_parts[0].numel() != rows * D:
        raise ValueError("pa_merge_partials: shape mismatch")
    if out is None:
        out = torch.empty(o_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
    if lse_out is None:
        lse_out = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
    _need(out, "out", torch.float32, o_parts.device)
    _need(lse_out, "lse_out", torch.float32, o_parts.device)
    st = _lib.load().pa_merge_partials(_ptr(o_parts), _ptr(lse_parts), n, rows, D,
                                       o_parts.stride(0) if n > 1 else 0,
                                       lse_parts.stride(0) if n > 1 else 0, _ptr(out),
                                       _ptr(lse_out), _stream(stream))
    _lib.check(st, "pa_merge_partials")
    return out, lse_out


def pa_validate_tables(block_tables: torch.Tensor, context_lens: torch.Tensor, num_pages: int,
                       page_size: int, d_err: torch.Tensor, stream=None) -> None:
    """OR PA_DERR_* bits into d_err (int32 device scalar) for bad tables."""
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32, block_tables.device)
    _need(d_err, "d_err", torch.int32, block_tables.device)
    st = _lib.load().pa_validate_tables(_ptr(block_tables), block_tables.shape[0],
                                        block_tables.shape[1], _ptr(context_lens), num_pages,
                                        page_size, _ptr(d_err), _stream(stream))
    _lib.check(st, "pa_validate_tables")
