"""Plain CPU oracle for paged decode attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its binding in ``paged_kv_cache_466_b200``) never imports it, and this package
imports nothing from the product. The two share only the seeded input
generators, which hold none of the method's arithmetic.

Contents, each written from the pages ("KV-Cache Optimization Techniques",
"Understanding KV-Cache Optimization in Modern LLM Serving"):

* ``scatter_rows``         — page-table resolution for writes: logical token
  ``pos`` of a sequence lives in physical page ``table[pos // P]`` at slot
  ``pos % P`` (section "PagedAttention (vLLM)", "Architecture").
* ``quantize_rows``        — Eq. 3 per-token INT8 quantiser (C, fp32 IEEE).
* ``quantize_rows_int4``   — per-token INT4 quantiser (Eq. 3 with 16 levels,
  two codes per byte).
* ``quantize_rows_fp8``    — per-token FP8 (E4M3) quantiser with an absmax scale
  (the pages' FP8 KV cache; encoding written from the format definition).
* ``paged_attention``      — Eq. 1 over gathered pages (C, fp64).
* ``paged_attention_window`` — Eq. 1 over the StreamingLLM token set of Eq. 5
  (attention sinks + last w tokens) / the sliding window of Eq. 6 (C, fp64).
* ``lse_merge``            — merging attention results of disjoint token
  ranges by their log-sum-exp. The pages do not describe split-KV; this is the
  plain identity softmax(x ∪ y) = weights exp(lse_x - M), exp(lse_y - M).
* ``eq2_*``                — Eq. 2 memory for N requests with a shared prefix
  (section "Prefix Caching"), in tokens and in pages.
* ``kv_memory_bytes``      — Memory_KV = 2 * L * H_kv * D * N * bytes (second
  page, "The Memory Math Behind KV-Cache").

Every function is pinned by tests in ``tests/test_oracle.py`` against values
the pages print, closed forms, or library routines; none is pinned against
the CUDA path.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_LIB = None


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the C oracle library."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_paged_attention.restype = ctypes.c_int
        L.oracle_paged_attention.argtypes = [
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_double, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_paged_attention_window.restype = ctypes.c_int
        L.oracle_paged_attention_window.argtypes = [
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_double, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_quantize_rows_fp8.restype = None
        L.oracle_quantize_rows_fp8.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                               ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_quantize_rows_int4.restype = None
        L.oracle_quantize_rows_int4.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                                ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_quantize_rows.restype = None
        L.oracle_quantize_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                           ctypes.c_void_p, ctypes.c_void_p]
        _LIB = L
    return _LIB


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# Eq. 3 quantiser
# --------------------------------------------------------------------------
def quantize_rows(x_bits: np.ndarray):
    """Per-row INT8 quantisation of bf16 rows (given as uint16 bit patterns).

    Returns ``codes`` (uint8, same shape) and ``sz`` (float32, [..., 2] with
    (scale, zero) per row). Eq. 3, "KV-Cache Quantization", per-token variant.
    """
    x = _c(x_bits, np.uint16)
    d = x.shape[-1]
    rows = x.reshape(-1, d)
    codes = np.empty(rows.shape, np.uint8)
    sz = np.empty((rows.shape[0], 2), np.float32)
    lib().oracle_quantize_rows(_ptr(rows), rows.shape[0], d, _ptr(codes), _ptr(sz))
    return codes.reshape(x.shape), sz.reshape(x.shape[:-1] + (2,))


def quantize_rows_fp8(x_bits: np.ndarray):
    """Per-row FP8 (E4M3) quantisation with an absmax fp32 scale (s = max|x|/448);
    returns codes (uint8 bit patterns) and sz [..., 2] = (s, 0)."""
    x = _c(x_bits, np.uint16)
    d = x.shape[-1]
    rows = x.reshape(-1, d)
    codes = np.empty(rows.shape, np.uint8)
    sz = np.empty((rows.shape[0], 2), np.float32)
    lib().oracle_quantize_rows_fp8(_ptr(rows), rows.shape[0], d, _ptr(codes), _ptr(sz))
    return codes.reshape(x.shape), sz.reshape(x.shape[:-1] + (2,))


def quantize_rows_int4(x_bits: np.ndarray):
    """Per-row INT4 quantisation (Eq. 3 with 16 levels); returns packed codes
    [..., D/2] (element 2i in the low nibble of byte i) and sz [..., 2]."""
    x = _c(x_bits, np.uint16)
    d = x.shape[-1]
    rows = x.reshape(-1, d)
    packed = np.empty((rows.shape[0], d // 2), np.uint8)
    sz = np.empty((rows.shape[0], 2), np.float32)
    lib().oracle_quantize_rows_int4(_ptr(rows), rows.shape[0], d, _ptr(packed), _ptr(sz))
    return packed.reshape(x.shape[:-1] + (d // 2,)), sz.reshape(x.shape[:-1] + (2,))


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """[..., D/2] bytes -> [..., D] codes (low nibble first)."""
    lo = packed & 15
    hi = packed >> 4
    return np.stack([lo, hi], -1).reshape(packed.shape[:-1] + (packed.shape[-1] * 2,))


def e4m3_value(code: int) -> float:
    return float(lib().oracle_e4m3_value(int(code)))


def e4m3_encode(r: float) -> int:
    return int(lib().oracle_e4m3_encode(float(r)))


# --------------------------------------------------------------------------
# Host pool and page-table resolution
# --------------------------------------------------------------------------
@dataclass
class HostPool:
    """A KV page pool in host memory: [num_pages][Hkv][P][D] per tensor."""
    kind: str                      # "bf16", "u8" (INT8, Eq. 3), "fp8" (E4M3) or "u4" (INT4)
    page_size: int
    k: np.ndarray                  # uint16 (bf16 bits) or uint8 codes
    v: np.ndarray
    k_sz: Optional[np.ndarray] = None   # float32 [num_pages][Hkv][P][2]
    v_sz: Optional[np.ndarray] = None

    @property
    def num_pages(self) -> int:
        return self.k.shape[0]

    @property
    def num_kv_heads(self) -> int:
        return self.k.shape[1]

    @property
    def head_dim(self) -> int:
        return self.k.shape[3] * (2 if self.kind == "u4" else 1)


def empty_pool(kind: str, num_pages: int, hkv: int, page_size: int, d: int,
               fill_byte: int = 0) -> HostPool:
    """A pool whose every byte is ``fill_byte`` (so untouched slots can be checked)."""
    if kind == "bf16":
        k = np.full((num_pages, hkv, page_size, d), fill_byte * 0x0101, np.uint16)
        return HostPool(kind, page_size, k, k.copy())
    if kind in ("u8", "fp8", "u4"):
        k = np.full((num_pages, hkv, page_size, d // 2 if kind == "u4" else d), fill_byte,
                    np.uint8)
        sz = np.frombuffer(bytes([fill_byte]) * (num_pages * hkv * page_size * 8),
                           np.float32).reshape(num_pages, hkv, page_size, 2).copy()
        return HostPool(kind, page_size, k, k.copy(), sz, sz.copy())
    raise ValueError(kind)


def scatter_rows(pool: HostPool, block_tables: np.ndarray, seq_idx: np.ndarray,
                 pos: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray) -> None:
    """Write token rows into their page slots; quantise first for an INT8 pool.

    Row i (shape [Hkv][D]) of sequence seq_idx[i] at logical position pos[i]
    goes to physical page block_tables[seq_idx[i]][pos[i] // P], slot
    pos[i] % P ("PagedAttention (vLLM)", "Architecture").
    """
    P = pool.page_size
    seq_idx = np.asarray(seq_idx, np.int64)
    pos = np.asarray(pos, np.int64)
    pages = np.asarray(block_tables)[seq_idx, pos // P].astype(np.int64)
    if np.any(pages < 0) or np.any(pages >= pool.num_pages):
        raise ValueError("page table entry outside the pool")
    slots = pos % P
    if pool.kind == "bf16":
        pool.k[pages, :, slots, :] = k_bits
        pool.v[pages, :, slots, :] = v_bits
    else:
        qf = {"u8": quantize_rows, "fp8": quantize_rows_fp8, "u4": quantize_rows_int4}[pool.kind]
        kc, ks = qf(k_bits)
        vc, vs = qf(v_bits)
        pool.k[pages, :, slots, :] = kc
        pool.v[pages, :, slots, :] = vc
        pool.k_sz[pages, :, slots, :] = ks
        pool.v_sz[pages, :, slots, :] = vs


# --------------------------------------------------------------------------
# Eq. 1 attention
# --------------------------------------------------------------------------
def paged_attention(pool: HostPool, q_bits: np.ndarray, block_tables: np.ndarray,
                    context_lens: np.ndarray, scale: float,
                    pairs: Optional[Sequence[Sequence[int]]] = None,
                    t_begin: int = 0, t_end: int = -1):
    """fp64 Eq. 1 for (b, hq) pairs (all if ``pairs`` is None).

    Returns (out [n, D] float64, lse [n] float64). ``t_begin``/``t_end``
    restrict every sequence to a token sub-range (``t_end < 0`` = whole context).
    """
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    assert D == pool.head_dim
    bt = _c(block_tables, np.int32)
    ctx = _c(context_lens, np.int32)
    pr = None if pairs is None else _c(np.asarray(pairs).reshape(-1, 2), np.int32)
    n = B * Hq if pr is None else pr.shape[0]
    out = np.zeros((n, D), np.float64)
    lse = np.zeros((n,), np.float64)
    kind = {"bf16": 0, "u8": 1, "fp8": 2, "u4": 3}[pool.kind]
    st = lib().oracle_paged_attention(
        kind, _ptr(_c(pool.k, pool.k.dtype)), _ptr(_c(pool.v, pool.v.dtype)),
        _ptr(None if pool.k_sz is None else _c(pool.k_sz, np.float32)),
        _ptr(None if pool.v_sz is None else _c(pool.v_sz, np.float32)),
        pool.num_pages, pool.page_size, pool.num_kv_heads, D, _ptr(q), B, Hq,
        _ptr(bt), bt.shape[1], _ptr(ctx), float(scale), int(t_begin), int(t_end),
        _ptr(pr), 0 if pr is None else pr.shape[0], _ptr(out), _ptr(lse))
    if st != 0:
        raise ValueError(f"oracle_paged_attention failed with status {st}")
    return out, lse


def paged_attention_window(pool: HostPool, q_bits: np.ndarray, block_tables: np.ndarray,
                           context_lens: np.ndarray, scale: float, sinks: int, window: int,
                           pairs: Optional[Sequence[Sequence[int]]] = None):
    """fp64 attention over {first `sinks`} U {last `window`} tokens of each
    sequence (Eq. 5; sinks = 0 is the sliding window of Eq. 6; window = 0
    means the whole context). Returns (out [n, D], lse [n])."""
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    bt = _c(block_tables, np.int32)
    ctx = _c(context_lens, np.int32)
    pr = None if pairs is None else _c(np.asarray(pairs).reshape(-1, 2), np.int32)
    n = B * Hq if pr is None else pr.shape[0]
    out = np.zeros((n, D), np.float64)
    lse = np.zeros((n,), np.float64)
    kind = {"bf16": 0, "u8": 1, "fp8": 2, "u4": 3}[pool.kind]
    st = lib().oracle_paged_attention_window(
        kind, _ptr(_c(pool.k, pool.k.dtype)), _ptr(_c(pool.v, pool.v.dtype)),
        _ptr(None if pool.k_sz is None else _c(pool.k_sz, np.float32)),
        _ptr(None if pool.v_sz is None else _c(pool.v_sz, np.float32)),
        pool.num_pages, pool.page_size, pool.num_kv_heads, D, _ptr(q), B, Hq,
        _ptr(bt), bt.shape[1], _ptr(ctx), float(scale), int(sinks), int(window),
        _ptr(pr), 0 if pr is None else pr.shape[0], _ptr(out), _ptr(lse))
    if st != 0:
        raise ValueError(f"oracle_paged_attention_window failed with status {st}")
    return out, lse


def lse_merge(o_parts: np.ndarray, lse_parts: np.ndarray) -> np.ndarray:
    """Merge normalised partial outputs of disjoint token ranges.

    o_parts [..., S, D], lse_parts [..., S] -> [..., D] in fp64:
    M = max_s lse_s; w_s = exp(lse_s - M); out = sum_s w_s o_s / sum_s w_s.
    A range with lse = -inf has weight 0; if every range is empty, out = 0.
    """
    o = np.asarray(o_parts, np.float64)
    lse = np.asarray(lse_parts, np.float64)
    M = np.max(lse, axis=-1, keepdims=True)
    finite = np.isfinite(M)
    Msafe = np.where(finite, M, 0.0)
    w = np.where(np.isfinite(lse), np.exp(lse - Msafe), 0.0)
    den = np.sum(w, axis=-1, keepdims=True)
    num = np.sum(w[..., None] * o, axis=-2)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), 0.0)


# --------------------------------------------------------------------------
# Eq. 2 and the memory formula
# --------------------------------------------------------------------------
def eq2_paged(n_requests: int, tokens_per_request: int, c: int = 1) -> int:
    """Eq. 2, left: Paged = N * T * c."""
    return n_requests * tokens_per_request * c


def eq2_prefix_cached(n_requests: int, tokens_per_request: int, p_shared: int,
                      c: int = 1) -> int:
    """Eq. 2, right: Prefix-cached = P_shared * c + N * (T - P_shared) * c."""
    return p_shared * c + n_requests * (tokens_per_request - p_shared) * c


def eq2_paged_var(lengths: Sequence[int], c: int = 1) -> int:
    """Eq. 2 (left) with per-request lengths T_i: sum_i T_i * c."""
    return sum(int(t) * c for t in lengths)


def eq2_prefix_cached_var(lengths: Sequence[int], p_shared: int, c: int = 1) -> int:
    """Eq. 2 (right) with per-request lengths: P_shared*c + sum_i (T_i - P_shared)*c."""
    return p_shared * c + sum((int(t) - p_shared) * c for t in lengths)


def eq2_pages_unshared(lengths: Sequence[int], page_size: int) -> int:
    """Pages when every request holds its own copy: sum_i ceil(T_i / P)."""
    return sum(-(-int(t) // page_size) for t in lengths)


def eq2_pages_shared(lengths: Sequence[int], p_shared: int, page_size: int) -> int:
    """Pages when a page-aligned prefix of p_shared tokens is stored once:
    p_shared / P + sum_i ceil((T_i - p_shared) / P)."""
    if p_shared % page_size:
        raise ValueError("the shared prefix must be page aligned")
    return p_shared // page_size + sum(-(-(int(t) - p_shared) // page_size) for t in lengths)


def kv_memory_bytes(layers: int, kv_heads: int, head_dim: int, tokens: int,
                    bytes_per_elem: float) -> float:
    """Memory_KV = 2 * L * H_kv * D * N * P_bytes (K and V, one request)."""
    v = 2 * layers * kv_heads * head_dim * tokens * bytes_per_elem
    return int(v) if float(v).is_integer() else v


def max_internal_waste_tokens(page_size: int) -> int:
    """Worst-case unused slots of one request under paging: its last page holds
    at least one token, so at most P - 1 slots are empty ("Benefits")."""
    return page_size - 1


