"""Context-parallel decode: one sequence's KV pages spread over several GPUs.

Rank r of a group of N holds the pages of tokens [r * T, (r + 1) * T) of every
sequence (the last rank also everything past N * T), T a multiple of the page
size. Each rank decodes its own range with ``pa_decode_range``; the normalised
partials and their log-sum-exps are all-gathered (one collective per decode
step, B * Hq * (D + 1) * 4 bytes from each rank, padded to 256 bytes) and every rank merges them
with ``pa_merge_partials``. The merge is the exact identity for a softmax over
disjoint token ranges (the split-KV merge of Eq. 1), so the result equals the
single-GPU decode up to fp32 rounding.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import KVPool, pa_decode_range, pa_merge_partials

_NO_END = 0x7FFFFFFF


def tokens_per_rank_for(max_context: int, world: int, page_size: int) -> int:
    """The even split of the longest context over ``world`` ranks, rounded up
    to whole pages (every rank but the last holds exactly this many tokens of
    a sequence that long)."""
    if max_context < 0 or world <= 0 or page_size <= 0:
        raise ValueError("bad max_context, world or page_size")
    per = -(-max(max_context, 1) // world)
    return -(-per // page_size) * page_size


def shard_tables(block_tables_width: int, context_lens, rank: int, world: int,
                 tokens_per_rank: int, page_size: int, seed: int = 0):
    """Rank ``rank``'s own page tables for a context-parallel layout: the
    logical pages of its token range get ids of a pool of its own (randomly
    permuted with ``seed``), every other entry is -1 (never read by the range
    decode). Returns (tables int32 [B, width], number of pages used)."""
    import numpy as np
    begin, end = rank_range(rank, world, tokens_per_rank)
    ctx = np.asarray(context_lens, dtype=np.int64)
    tables = np.full((len(ctx), block_tables_width), -1, np.int32)
    lp_begin = begin // page_size
    want = []
    for b, c in enumerate(ctx.tolist()):
        hi = -(-c // page_size)
        if end != _NO_END:
            hi = min(hi, end // page_size)
        want += [(b, lp) for lp in range(lp_begin, hi)]
    ids = np.random.default_rng(seed).permutation(len(want)).astype(np.int32)
    for (b, lp), pid in zip(want, ids.tolist()):
        tables[b, lp] = pid
    return tables, len(want)


def rank_range(rank: int, world: int, tokens_per_rank: int) -> Tuple[int, int]:
    """Token range [begin, end) rank ``rank`` of ``world`` decodes."""
    if tokens_per_rank <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank or tokens_per_rank")
    begin = rank * tokens_per_rank
    end = _NO_END if rank == world - 1 else begin + tokens_per_rank
    return begin, end


def partial_block_floats(num_seqs: int, num_q_heads: int, head_dim: int) -> int:
    """fp32 words one rank contributes to the all-gather: its o [B, Hq, D]
    then its lse [B, Hq], padded to 64 words so every rank's block starts on a
    256-byte boundary of the gathered buffer."""
    rows = num_seqs * num_q_heads
    return (rows * (head_dim + 1) + 63) // 64 * 64


def partial_views(block: torch.Tensor, num_seqs: int, num_q_heads: int, head_dim: int):
    """(o [B, Hq, D], lse [B, Hq]) views into one rank's block."""
    rows = num_seqs * num_q_heads
    o = block[:rows * head_dim].view(num_seqs, num_q_heads, head_dim)
    lse = block[rows * head_dim:rows * (head_dim + 1)].view(num_seqs, num_q_heads)
    return o, lse


def gathered_views(gathered: torch.Tensor, world: int, num_seqs: int, num_q_heads: int,
                   head_dim: int):
    """(o_parts [world, B, Hq, D], lse_parts [world, B, Hq]) strided views into
    the all-gathered buffer, ready for ``pa_merge_partials``."""
    rows = num_seqs * num_q_heads
    per = gathered.view(world, -1)
    o = per[:, :rows * head_dim].view(world, num_seqs, num_q_heads, head_dim)
    lse = per[:, rows * head_dim:rows * (head_dim + 1)].view(world, num_seqs, num_q_heads)
    return o, lse


def decode_context_parallel(pool: KVPool, q: torch.Tensor, block_tables: torch.Tensor,
                            context_lens: torch.Tensor, scale: float, tokens_per_rank: int,
                            group: Optional[dist.ProcessGroup] = None,
                            out: Optional[torch.Tensor] = None, num_splits: int = 0,
                            d_err: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Eq. 1 for every (sequence, query head) with the KV pages of token range
    ``rank_range(rank, world, tokens_per_rank)`` on this rank (its pool and
    tables; entries outside the range are not read). Every rank gets the full
    output. ``tokens_per_rank`` must be a multiple of the page size.

    The range's o and lse are written straight into this rank's block of one
    fp32 buffer, so a single all-gather moves both, and the merge reads the
    gathered buffer in place. Without an initialised process group the call
    is the one-rank case (the whole context on this GPU, no collective)."""
    if dist.is_available() and dist.is_initialized():
        rank = dist.get_rank(group)
        world = dist.get_world_size(group)
    else:
        rank, world = 0, 1
    if tokens_per_rank % pool.page_size != 0:
        raise ValueError("tokens_per_rank must be a multiple of the page size")
    B, Hq, D = q.shape
    begin, end = rank_range(rank, world, tokens_per_rank)
    block = torch.empty(partial_block_floats(B, Hq, D), dtype=torch.float32, device=q.device)
    o, lse = partial_views(block, B, Hq, D)
    pa_decode_range(pool, q, block_tables, context_lens, scale, begin, end, o_out=o,
                    lse_out=lse, num_splits=num_splits, d_err=d_err)
    if world == 1:
        gathered = block
    else:
        gathered = torch.empty(world * block.numel(), dtype=torch.float32, device=q.device)
        dist.all_gather_into_tensor(gathered, block, group=group)
    o_parts, lse_parts = gathered_views(gathered, world, B, Hq, D)
    merged, _ = pa_merge_partials(o_parts, lse_parts, out=out)
    return merged


__all__ = ["rank_range", "tokens_per_rank_for", "shard_tables", "partial_block_floats", "partial_views", "gathered_views",
           "decode_context_parallel"]
