"""Host-side page bookkeeping for the paged KV cache.

"KV-Cache Optimization Techniques", section "PagedAttention (vLLM)",
"Architecture": the pool is divided into pages of P tokens, each request has a
page table, pages are allocated only when needed and freed when the request
completes; "Prefix Caching": requests with a common prefix reuse the prefix's
pages. This module keeps that bookkeeping on the host (a free list with
reference counts) and produces the int32 block tables the kernels read. It
does no attention arithmetic; the device only ever sees the tables.
"""
from __future__ import annotations

from typing import Dict, Iterable, List, Optional, Sequence

import numpy as np


def pages_for(tokens: int, page_size: int) -> int:
    """Pages a request of ``tokens`` tokens occupies: ceil(tokens / P)."""
    return -(-int(tokens) // page_size)


def kv_bytes(layers: int, kv_heads: int, head_dim: int, tokens: int,
             bytes_per_elem: float) -> float:
    """KV-cache size of one request: 2 (K and V) * L * H_kv * D * N * bytes
    ("Understanding KV-Cache Optimization in Modern LLM Serving", "The Memory
    Math Behind KV-Cache")."""
    v = 2 * layers * kv_heads * head_dim * tokens * bytes_per_elem
    return int(v) if float(v).is_integer() else v


def pool_bytes(num_pages: int, kv_heads: int, page_size: int, head_dim: int,
               kind: str = "bf16") -> int:
    """Device bytes of one layer's pool in this library's layout: K and V,
    each row ``head_dim`` bf16 values, or for the quantised caches its codes
    (one byte per element for INT8 and FP8, two elements per byte for INT4)
    plus the row's fp32 (scale, zero)."""
    rows = num_pages * kv_heads * page_size
    if kind == "bf16":
        return 2 * rows * head_dim * 2
    if kind in ("u8", "fp8"):
        return 2 * rows * (head_dim + 8)
    if kind == "u4":
        if head_dim % 2:
            raise ValueError("an INT4 row packs two elements per byte: head_dim must be even")
        return 2 * rows * (head_dim // 2 + 8)
    raise ValueError(f"unknown cache kind {kind!r}")


class OutOfPages(RuntimeError):
    pass


class PageAllocator:
    """Free list of physical page ids with reference counts.

    A page returns to the free list when its last reference is released, so a
    prefix page shared by several requests lives as long as any of them.
    """

    def __init__(self, num_pages: int, order: Optional[Iterable[int]] = None):
        self.num_pages = int(num_pages)
        ids = list(range(num_pages)) if order is None else [int(i) for i in order]
        if sorted(ids) != list(range(num_pages)):
            raise ValueError("order must be a permutation of the page ids")
        self._free: List[int] = ids[::-1]           # pop() hands out ids[0] first
        self._ref = np.zeros(num_pages, np.int32)

    @property
    def free_pages(self) -> int:
        return len(self._free)

    @property
    def used_pages(self) -> int:
        return self.num_pages - len(self._free)

    def alloc(self) -> int:
        if not self._free:
            raise OutOfPages("page pool exhausted")
        p = self._free.pop()
        self._ref[p] = 1
        return p

    def retain(self, page: int) -> None:
        if self._ref[page] <= 0:
            raise ValueError(f"page {page} is not allocated")
        self._ref[page] += 1

    def release(self, page: int) -> None:
        if self._ref[page] <= 0:
            raise ValueError(f"page {page} released twice")
        self._ref[page] -= 1
        if self._ref[page] == 0:
            self._free.append(page)

    def refcount(self, page: int) -> int:
        return int(self._ref[page])


class Request:
    """One sequence's page table and length."""

    def __init__(self, alloc: PageAllocator, page_size: int):
        self.alloc = alloc
        self.P = page_size
        self.pages: List[int] = []
        self.length = 0

    def share_prefix(self, other: "Request", tokens: int) -> None:
        """Point this (empty) request's first tokens at ``other``'s pages.

        Only whole pages are shared, so ``tokens`` must be a multiple of P and
        later appends never write into a shared page (no copy-on-write needed).
        """
        if self.length or self.pages:
            raise ValueError("share_prefix needs an empty request")
        if tokens % self.P or tokens > other.length:
            raise ValueError("a shared prefix must be whole pages of the other request")
        for p in other.pages[:tokens // self.P]:
            self.alloc.retain(p)
            self.pages.append(p)
        self.length = tokens

    def append(self, n: int = 1) -> List[tuple]:
        """Reserve slots for n new tokens, allocating pages on demand.

        Returns the (position, page, slot) of each new token.
        """
        out = []
        for _ in range(n):
            pos = self.length
            if pos // self.P == len(self.pages):
                self.pages.append(self.alloc.alloc())
            page = self.pages[pos // self.P]
            if self.alloc.refcount(page) > 1:
                raise ValueError("append into a shared page: copy-on-write is the caller's job")
            out.append((pos, page, pos % self.P))
            self.length += 1
        return out

    def release(self) -> None:
        for p in self.pages:
            self.alloc.release(p)
        self.pages = []
        self.length = 0

    @property
    def wasted_slots(self) -> int:
        """Allocated but unused token slots (at most P - 1)."""
        return len(self.pages) * self.P - self.length


def block_tables(requests: Sequence[Request], max_pages: Optional[int] = None) -> np.ndarray:
    """int32 [B, max_pages] table, -1 past each request's pages."""
    width = max_pages if max_pages is not None else max([len(r.pages) for r in requests] + [1])
    t = np.full((len(requests), width), -1, np.int32)
    for i, r in enumerate(requests):
        if len(r.pages) > width:
            raise ValueError("request has more pages than the table width")
        t[i, :len(r.pages)] = r.pages
    return t


def pages_in_use(requests: Sequence[Request]) -> int:
    """Distinct physical pages referenced by the requests."""
    seen: Dict[int, None] = {}
    for r in requests:
        for p in r.pages:
            seen[p] = None
    return len(seen)
