"""Seeded synthetic decode workloads (inputs only).

This module draws the inputs that both the CUDA path and the CPU oracle
consume: context lengths, physical page ids, block tables, the query rows and
the K/V token rows to be written into the cache. It holds none of the method's
arithmetic — no page-slot resolution, no quantisation, no attention — so it can
feed both sides without coupling them.

Every draw comes from one CPU ``torch.Generator`` seeded with ``seed`` (0 by
default), in this order: context lengths -> physical page permutation -> q ->
K rows (sequence by sequence) -> V rows -> outlier masks and values. Values are
drawn in fp32 and rounded once to bf16.

The five workloads mirror the decode shapes the pages discuss (Llama-3-8B- and
70B-shaped GQA layers, an INT8 cache, a shared system-prompt prefix):

* ``tiny``      B=4, ctx {1,17,33,64}, Hq=4, Hkv=2, D=64, P=16, 32-page pool
* ``llama8b``   B=64, ctx ~ U{128..4096}, Hq=32, Hkv=8, D=128, P=16, pool = 1.1 x need
* ``llama70b``  B=32, ctx = 8192, Hq=64, Hkv=8, D=128, P=32, 8192-page pool (1.07 GB)
* ``int8``      ``llama8b`` draws + 1 % outliers ~ N(0, 8^2), stored as per-token INT8
* ``prefix``    128 requests sharing a 2000-token (125-page) prefix + U{1..512} suffix

Each sequence's last token is the "step" token, appended through the cache
write before decoding; all earlier tokens form the prefill list.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    P: int
    kv: str                         # "bf16", "u8" (INT8), "fp8" (E4M3) or "u4" (INT4)
    num_pages: int
    max_pages: int
    scale: float
    context_lens: np.ndarray        # int32 [B]
    block_tables: np.ndarray        # int32 [B, max_pages], -1 where unused
    q: torch.Tensor                 # bf16 [B, Hq, D]
    prefill_seq: np.ndarray         # int32 [N]
    prefill_pos: np.ndarray         # int32 [N]
    prefill_k: torch.Tensor         # bf16 [N, Hkv, D]
    prefill_v: torch.Tensor
    step_seq: np.ndarray            # int32 [B']
    step_pos: np.ndarray
    step_k: torch.Tensor            # bf16 [B', Hkv, D]
    step_v: torch.Tensor
    notes: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def total_tokens(self) -> int:
        return int(self.context_lens.astype(np.int64).sum())

    def all_rows(self):
        """Prefill and step rows together, in write order."""
        return (np.concatenate([self.prefill_seq, self.step_seq]),
                np.concatenate([self.prefill_pos, self.step_pos]),
                torch.cat([self.prefill_k, self.step_k]),
                torch.cat([self.prefill_v, self.step_v]))

    def step_rows_by_sequence(self):
        """The step rows laid out per sequence, as pa_decode_append takes them:
        (k_new, v_new) bf16 [B, Hkv, D] with row b = sequence b's step token
        and zeros for a sequence without one; None unless every step row is
        its sequence's newest position (ctx_b - 1) and every sequence with
        ctx_b >= 1 has one."""
        ctx = self.context_lens
        if len(set(self.step_seq.tolist())) != len(self.step_seq):
            return None
        if not np.array_equal(np.sort(self.step_seq), np.flatnonzero(ctx >= 1)):
            return None
        if not np.array_equal(self.step_pos, ctx[self.step_seq] - 1):
            return None
        k = torch.zeros((self.B, self.Hkv, self.D), dtype=torch.bfloat16)
        v = torch.zeros_like(k)
        idx = torch.from_numpy(self.step_seq.astype(np.int64))
        k[idx] = self.step_k
        v[idx] = self.step_v
        return k, v


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 array of its bit patterns (no copy if possible)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _randn_bf16(g: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def _with_outliers(g: torch.Generator, x: torch.Tensor, frac: float, sigma: float) -> torch.Tensor:
    """Replace a Bernoulli(frac) subset of elements by N(0, sigma^2) draws."""
    if frac <= 0:
        return x
    mask = torch.rand(x.shape, generator=g) < frac
    vals = torch.randn(x.shape, generator=g, dtype=torch.float32) * sigma
    return torch.where(mask, vals, x.float()).to(torch.bfloat16)


def _assemble(name, B, Hq, Hkv, D, P, kv, num_pages, max_pages, ctx, tables, q,
              seqs_k, seqs_v, first_pos, notes) -> Workload:
    """Build the prefill/step lists from per-sequence token rows.

    ``seqs_k[b]`` holds the rows of sequence b starting at logical position
    ``first_pos[b]`` (positions before that are written by another sequence's
    rows, e.g. a shared prefix). The last position of each sequence is the
    step token.
    """
    pre_seq, pre_pos, pre_k, pre_v = [], [], [], []
    st_seq, st_pos, st_k, st_v = [], [], [], []
    for b in range(B):
        kb, vb = seqs_k[b], seqs_v[b]
        n = kb.shape[0]
        if n == 0:
            continue
        p0 = first_pos[b]
        last = p0 + n - 1
        if last == ctx[b] - 1:
            st_seq.append(b)
            st_pos.append(last)
            st_k.append(kb[-1:])
            st_v.append(vb[-1:])
            kb, vb, n = kb[:-1], vb[:-1], n - 1
        pre_seq.append(np.full(n, b, np.int32))
        pre_pos.append(np.arange(p0, p0 + n, dtype=np.int32))
        pre_k.append(kb)
        pre_v.append(vb)
    e = torch.zeros((0, Hkv, D), dtype=torch.bfloat16)
    return Workload(
        name=name, B=B, Hq=Hq, Hkv=Hkv, D=D, P=P, kv=kv, num_pages=num_pages,
        max_pages=max_pages, scale=1.0 / math.sqrt(D),
        context_lens=np.asarray(ctx, np.int32), block_tables=tables, q=q,
        prefill_seq=np.concatenate(pre_seq) if pre_seq else np.zeros(0, np.int32),
        prefill_pos=np.concatenate(pre_pos) if pre_pos else np.zeros(0, np.int32),
        prefill_k=torch.cat(pre_k) if pre_k else e, prefill_v=torch.cat(pre_v) if pre_v else e,
        step_seq=np.asarray(st_seq, np.int32), step_pos=np.asarray(st_pos, np.int32),
        step_k=torch.cat(st_k) if st_k else e, step_v=torch.cat(st_v) if st_v else e,
        notes=notes)


def paged(name: str, *, B: int, Hq: int, Hkv: int, D: int, P: int,
          context_lens: Optional[Sequence[int]] = None, ctx_range=(128, 4096),
          pool_pages: Optional[int] = None, pool_slack: float = 0.0,
          max_pages: Optional[int] = None, kv: str = "bf16",
          outlier_frac: float = 0.0, outlier_sigma: float = 8.0,
          seed: int = 0) -> Workload:
    """A batch of independent sequences in one randomly permuted page pool.

    Pages needed by sequence b: ceil(ctx_b / P). The pool has ``pool_pages``
    pages (default: ceil((1 + pool_slack) * need)); a random permutation of the
    pool's ids is dealt out in (sequence, logical page) order.
    """
    g = torch.Generator().manual_seed(seed)
    if context_lens is None:
        lo, hi = ctx_range
        ctx = torch.randint(lo, hi + 1, (B,), generator=g).tolist()
    else:
        ctx = [int(c) for c in context_lens]
        assert len(ctx) == B
    npg = [-(-c // P) for c in ctx]
    need = sum(npg)
    if pool_pages is None:
        pool_pages = max(1, math.ceil((1.0 + pool_slack) * need))
    assert pool_pages >= need
    if max_pages is None:
        max_pages = max(1, max(npg) if npg else 1)
    perm = torch.randperm(pool_pages, generator=g).numpy().astype(np.int32)
    tables = np.full((B, max_pages), -1, np.int32)
    k = 0
    for b in range(B):
        tables[b, :npg[b]] = perm[k:k + npg[b]]
        k += npg[b]
    q = _randn_bf16(g, (B, Hq, D))
    ks = [_randn_bf16(g, (c, Hkv, D)) for c in ctx]
    vs = [_randn_bf16(g, (c, Hkv, D)) for c in ctx]
    if outlier_frac > 0:
        ks = [_with_outliers(g, x, outlier_frac, outlier_sigma) for x in ks]
        vs = [_with_outliers(g, x, outlier_frac, outlier_sigma) for x in vs]
    return _assemble(name, B, Hq, Hkv, D, P, kv, pool_pages, max_pages, ctx, tables, q,
                     ks, vs, [0] * B, {"need_pages": need, "seed": seed})


def tiny(seed: int = 0) -> Workload:
    """B=4, ctx {1,17,33,64}, Hq=4, Hkv=2, D=64, P=16, 32-page pool."""
    return paged("tiny", B=4, Hq=4, Hkv=2, D=64, P=16, context_lens=[1, 17, 33, 64],
                 pool_pages=32, seed=seed)


def llama8b(B: int = 64, ctx_range=(128, 4096), seed: int = 0, kv: str = "bf16",
            outlier_frac: float = 0.0) -> Workload:
    """Llama-3-8B-shaped layer: Hq=32, Hkv=8, D=128, P=16, pool = 1.1 x need."""
    return paged({"bf16": "llama8b", "u8": "int8", "fp8": "fp8", "u4": "int4"}[kv], B=B, Hq=32,
                 Hkv=8, D=128, P=16,
                 ctx_range=ctx_range, pool_slack=0.10, max_pages=-(-ctx_range[1] // 16),
                 kv=kv, outlier_frac=outlier_frac, seed=seed)


def llama70b(B: int = 32, ctx: int = 8192, seed: int = 0) -> Workload:
    """Llama-3-70B-shaped long-context layer: Hq=64, Hkv=8, D=128, P=32,
    every context 8192 tokens, pool exactly the 8192 pages needed (B=32)."""
    return paged("llama70b", B=B, Hq=64, Hkv=8, D=128, P=32, context_lens=[ctx] * B,
                 seed=seed)


def fp8(B: int = 64, ctx_range=(128, 4096), seed: int = 0) -> Workload:
    """``llama8b`` draws plus 1 % outliers ~ N(0, 8^2), cached as per-token FP8 (E4M3)."""
    w = llama8b(B=B, ctx_range=ctx_range, seed=seed, kv="fp8", outlier_frac=0.01)
    w.name = "fp8"
    return w


def int4(B: int = 64, ctx_range=(128, 4096), seed: int = 0) -> Workload:
    """``llama8b`` draws plus 1 % outliers ~ N(0, 8^2), cached as per-token INT4."""
    return llama8b(B=B, ctx_range=ctx_range, seed=seed, kv="u4", outlier_frac=0.01)


def int8(B: int = 64, ctx_range=(128, 4096), seed: int = 0) -> Workload:
    """``llama8b`` draws plus 1 % outliers ~ N(0, 8^2), cached as per-token INT8."""
    return llama8b(B=B, ctx_range=ctx_range, seed=seed, kv="u8", outlier_frac=0.01)


def prefix(B: int = 128, prefix_tokens: int = 2000, suffix_range=(1, 512), Hq: int = 32,
           Hkv: int = 8, D: int = 128, P: int = 16, seed: int = 0):
    """Requests sharing one page-aligned prefix, each with its own suffix.

    Returns (shared, unshared): the same token values, once with every block
    table pointing at the same ``prefix_tokens / P`` physical prefix pages and
    once with a private copy of the prefix per request.
    """
    assert prefix_tokens % P == 0
    g = torch.Generator().manual_seed(seed)
    lo, hi = suffix_range
    suf = torch.randint(lo, hi + 1, (B,), generator=g).tolist()
    ctx = [prefix_tokens + s for s in suf]
    n_pre = prefix_tokens // P
    n_suf = [-(-s // P) for s in suf]
    max_pages = n_pre + -(-hi // P)
    # shared pool
    num_pages = n_pre + sum(n_suf)
    perm = torch.randperm(num_pages, generator=g).numpy().astype(np.int32)
    pre_ids = perm[:n_pre]
    tables = np.full((B, max_pages), -1, np.int32)
    k = n_pre
    for b in range(B):
        tables[b, :n_pre] = pre_ids
        tables[b, n_pre:n_pre + n_suf[b]] = perm[k:k + n_suf[b]]
        k += n_suf[b]
    q = _randn_bf16(g, (B, Hq, D))
    pk = _randn_bf16(g, (prefix_tokens, Hkv, D))
    sk = [_randn_bf16(g, (s, Hkv, D)) for s in suf]
    pv = _randn_bf16(g, (prefix_tokens, Hkv, D))
    sv = [_randn_bf16(g, (s, Hkv, D)) for s in suf]
    # shared: request 0 writes the prefix once; every request writes its suffix
    seqs_k = [torch.cat([pk, sk[0]])] + sk[1:]
    seqs_v = [torch.cat([pv, sv[0]])] + sv[1:]
    first = [0] + [prefix_tokens] * (B - 1)
    shared = _assemble("prefix", B, Hq, Hkv, D, P, "bf16", num_pages, max_pages, ctx,
                       tables, q, seqs_k, seqs_v, first,
                       {"prefix_tokens": prefix_tokens, "suffix": suf, "seed": seed,
                        "prefix_pages": pre_ids.copy()})
    # unshared copy: every request holds its own prefix pages (own permutation)
    g2 = torch.Generator().manual_seed(seed + 1)
    num_pages_u = B * n_pre + sum(n_suf)
    perm_u = torch.randperm(num_pages_u, generator=g2).numpy().astype(np.int32)
    tables_u = np.full((B, max_pages), -1, np.int32)
    k = 0
    for b in range(B):
        n = n_pre + n_suf[b]
        tables_u[b, :n] = perm_u[k:k + n]
        k += n
    seqs_k_u = [torch.cat([pk, sk[b]]) for b in range(B)]
    seqs_v_u = [torch.cat([pv, sv[b]]) for b in range(B)]
    unshared = _assemble("prefix-unshared", B, Hq, Hkv, D, P, "bf16", num_pages_u,
                         max_pages, ctx, tables_u, q, seqs_k_u, seqs_v_u, [0] * B,
                         {"prefix_tokens": prefix_tokens, "suffix": suf, "seed": seed})
    return shared, unshared


def by_name(name: str, **kw):
    """Full-size workload by name (``prefix`` returns the shared variant)."""
    if name == "tiny":
        return tiny(**kw)
    if name == "llama8b":
        return llama8b(**kw)
    if name == "llama70b":
        return llama70b(**kw)
    if name == "int8":
        return int8(**kw)
    if name == "fp8":
        return fp8(**kw)
    if name == "int4":
        return int4(**kw)
    if name == "prefix":
        return prefix(**kw)[0]
    raise KeyError(name)


__all__ = ["Workload", "bits", "paged", "tiny", "llama8b", "llama70b", "int8", "fp8", "int4",
           "prefix",
           "by_name"]
