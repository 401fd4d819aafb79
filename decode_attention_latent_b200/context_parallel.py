"""Context-parallel decode: every sequence's KV cache split by length across ranks.

Rank r of W holds a contiguous range of each sequence's pages, runs the decode
(``mla_decode``) on that range alone, and the W partial states (out, lse) are
gathered over ``torch.distributed`` and merged through their log-sum-exps by
``mla_merge_states``.  The merge is the online softmax of "FlashMLA:
compressing the KV cache" (jsqmd.com), "compute flow", step 4, applied to
whole partial results.  Splitting attention over devices by sequence length
is the idea of Ring Attention, which the FlashMLA-ETAP paper's page on
mlsanity.com lists under "Builds on"; decode needs no ring, since the query is
one token: one exchange per step, an all-gather of W x B x H x (1 KB + 4 B),
and no collective inside the attention itself.

Queries of s_q > 1 tokens: query position i sees the first L - s_q + 1 + i
tokens, so only the last s_q - 1 tokens of a sequence are hidden from some
position.  The split keeps all of them on the last rank (its first page is
moved down to the page holding token L - s_q + 1 when the balanced cut would
fall after it), which runs the causal decode on its shard: the kernel hides
the last s_q - 1 - i tokens of that shard, the right ones.  Every other rank
holds only tokens that all query positions see, so it folds the positions
into the heads -- q as [B, 1, s_q H, 576], an unmasked decode that still reads
each cache tile once -- and unfolds the result.  That needs s_q H <= 128.
"""
from __future__ import annotations

import contextlib
from typing import Callable, List, Optional, Tuple

import torch
import torch.distributed as dist

from . import decode, merge_states, PAGE


def page_cuts(num_pages: int, world_size: int, rank: int) -> Tuple[int, int]:
    """Pages [p0, p1) of a sequence with ``num_pages`` pages that rank
    ``rank`` of ``world_size`` holds: contiguous, balanced to one page."""
    if not 0 <= rank < world_size:
        raise ValueError("rank must be in [0, world_size)")
    return num_pages * rank // world_size, num_pages * (rank + 1) // world_size


def sequence_cuts(seqlen: int, world_size: int, rank: int, s_q: int = 1) -> Tuple[int, int]:
    """Pages [p0, p1) of one sequence of ``seqlen`` tokens on rank ``rank``:
    the balanced ``page_cuts``, except that for s_q > 1 no rank but the last
    ends after the page holding token seqlen - s_q + 1, the first token some
    query position does not see (so all such tokens are on the last rank)."""
    if s_q < 1:
        raise ValueError("s_q must be positive")
    pages = (seqlen + PAGE - 1) // PAGE
    p0, p1 = page_cuts(pages, world_size, rank)
    if s_q > 1:
        bound = max(0, seqlen - s_q + 1) // PAGE
        p0 = min(p0, bound) if rank > 0 else 0
        p1 = pages if rank == world_size - 1 else min(p1, bound)
    return p0, p1


def local_shard(cache_seqlens: torch.Tensor, block_table: torch.Tensor, world_size: int,
                rank: int, s_q: int = 1) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's view of a globally paged batch: (local lengths int32 [B],
    local page table int32 [B, max local pages]) on the inputs' device.  Page
    j of sequence b on this rank is global page p0(b) + j, so the local table
    still names blocks of the cache it was built for; a serving system that
    keeps each rank's pages in that rank's own cache builds the same local
    lengths with its own block ids.  ``s_q``: the query tokens per sequence
    (``sequence_cuts``)."""
    if cache_seqlens.dim() != 1 or block_table.dim() != 2 or block_table.shape[0] != cache_seqlens.shape[0]:
        raise ValueError("cache_seqlens must be [B] and block_table [B, max_blocks]")
    lens = cache_seqlens.detach().to("cpu", torch.int64).tolist()
    table = block_table.detach().to("cpu")
    cuts = []
    for L in lens:
        if L < 0:
            raise ValueError("negative sequence length")
        cuts.append(sequence_cuts(L, world_size, rank, s_q))
    width = max(1, max(p1 - p0 for p0, p1 in cuts))
    local_table = torch.zeros(len(lens), width, dtype=torch.int32)
    local_lens = torch.zeros(len(lens), dtype=torch.int32)
    for b, (L, (p0, p1)) in enumerate(zip(lens, cuts)):
        if p1 > table.shape[1]:
            raise ValueError(f"sequence {b} needs {p1} pages but the table has {table.shape[1]}")
        local_table[b, :p1 - p0] = table[b, p0:p1]
        local_lens[b] = max(0, min(L, PAGE * p1) - PAGE * p0)
    return local_lens.to(cache_seqlens.device), local_table.to(block_table.device)


def gather_states(out: torch.Tensor, lse: torch.Tensor,
                  group: Optional[dist.ProcessGroup] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gather every rank's partial state: (out [W, ...], lse [W, ...]) in
    rank order.  NCCL gathers straight into the stacked buffers; other
    backends gather a list (out travels as its bytes)."""
    W = dist.get_world_size(group)
    out_parts = torch.empty((W,) + tuple(out.shape), dtype=out.dtype, device=out.device)
    lse_parts = torch.empty((W,) + tuple(lse.shape), dtype=lse.dtype, device=lse.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out_parts, out.contiguous(), group=group)
        dist.all_gather_into_tensor(lse_parts, lse.contiguous(), group=group)
        return out_parts, lse_parts
    carrier = out.contiguous().view(torch.uint8)
    pieces = [torch.empty_like(carrier) for _ in range(W)]
    dist.all_gather(pieces, carrier, group=group)
    torch.stack(pieces, out=out_parts.view(torch.uint8))
    lse_pieces = [torch.empty_like(lse) for _ in range(W)]
    dist.all_gather(lse_pieces, lse.contiguous(), group=group)
    torch.stack(lse_pieces, out=lse_parts)
    return out_parts, lse_parts


def check_query_shape(q: torch.Tensor) -> None:
    """The shapes every rank accepts alike (a refusal on one rank only would
    leave the others waiting in the exchange): q [B, s_q, H, 576] with s_q H
    at most 128 when s_q > 1 (the folded query of the ranks before the last)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, s_q, H, 576]")
    s_q, H = q.shape[1], q.shape[2]
    if s_q > 1 and s_q * H > 128:
        raise ValueError("context-parallel decode with s_q > 1 needs s_q x H <= 128")


def query_view(q: torch.Tensor, last_rank: bool) -> Tuple[torch.Tensor, Callable]:
    """The query this rank decodes and the map of its (out, lse) back to
    [B, s_q, H, ...]: the causal query itself on the last rank (and for
    s_q = 1), else the positions folded into heads, [B, 1, s_q H, 576]."""
    B, s_q, H = q.shape[0], q.shape[1], q.shape[2]
    if s_q == 1 or last_rank:
        return q, lambda out, lse: (out, lse)
    return q.reshape(B, 1, s_q * H, q.shape[3]), lambda out, lse: (out.view(B, s_q, H, out.shape[-1]),
                                                                     lse.view(B, s_q, H))


def decode_local_state(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor,
                       cache_seqlens: torch.Tensor, softmax_scale: float, last_rank: bool) -> List[torch.Tensor]:
    """This rank's partial state (out bf16 [B, s_q, H, 512], lse fp32
    [B, s_q, H]) over its shard (``local_shard`` with the same s_q)."""
    check_query_shape(q)
    qv, back = query_view(q, last_rank)
    out, lse = decode(qv, kv_cache, block_table, cache_seqlens, softmax_scale)
    return list(back(out, lse))


def decode_context_parallel(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor,
                            cache_seqlens: torch.Tensor, softmax_scale: float, *,
                            group: Optional[dist.ProcessGroup] = None,
                            stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One decode step of a context-parallel group: ``kv_cache``,
    ``block_table`` and ``cache_seqlens`` describe this rank's pages of every
    sequence (``local_shard``, with the query's s_q); ``q`` is the same on
    every rank.  Returns the merged (out bf16 [B, s_q, H, 512], lse fp32
    [B, s_q, H]) on every rank."""
    check_query_shape(q)
    W = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    # the collective runs on the current stream: make `stream` current for all three steps
    with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
        out, lse = decode_local_state(q, kv_cache, block_table, cache_seqlens, softmax_scale, rank == W - 1)
        if not dist.is_initialized():
            return out, lse
        out_parts, lse_parts = gather_states(out, lse, group)
        return merge_states(out_parts, lse_parts)
