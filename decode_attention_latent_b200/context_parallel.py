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

Only single-token queries (s_q = 1) are split this way: with s_q > 1 the
causal window of query i ends s_q - 1 - i tokens before the sequence end, so
every rank but the last would need the whole sequence's length to place it.
"""
from __future__ import annotations

import contextlib
from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import decode, merge_states, PAGE


def page_cuts(num_pages: int, world_size: int, rank: int) -> Tuple[int, int]:
    """Pages [p0, p1) of a sequence with ``num_pages`` pages that rank
    ``rank`` of ``world_size`` holds: contiguous, balanced to one page."""
    if not 0 <= rank < world_size:
        raise ValueError("rank must be in [0, world_size)")
    return num_pages * rank // world_size, num_pages * (rank + 1) // world_size


def local_shard(cache_seqlens: torch.Tensor, block_table: torch.Tensor, world_size: int,
                rank: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's view of a globally paged batch: (local lengths int32 [B],
    local page table int32 [B, max local pages]) on the inputs' device.  Page
    j of sequence b on this rank is global page p0(b) + j, so the local table
    still names blocks of the cache it was built for; a serving system that
    keeps each rank's pages in that rank's own cache builds the same local
    lengths with its own block ids."""
    if cache_seqlens.dim() != 1 or block_table.dim() != 2 or block_table.shape[0] != cache_seqlens.shape[0]:
        raise ValueError("cache_seqlens must be [B] and block_table [B, max_blocks]")
    lens = cache_seqlens.detach().to("cpu", torch.int64).tolist()
    table = block_table.detach().to("cpu")
    cuts = []
    for L in lens:
        if L < 0:
            raise ValueError("negative sequence length")
        cuts.append(page_cuts((L + PAGE - 1) // PAGE, world_size, rank))
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


def decode_context_parallel(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor,
                            cache_seqlens: torch.Tensor, softmax_scale: float, *,
                            group: Optional[dist.ProcessGroup] = None,
                            stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One decode step of a context-parallel group: ``kv_cache``,
    ``block_table`` and ``cache_seqlens`` describe this rank's pages of every
    sequence (``local_shard``); ``q`` is the same on every rank.  Returns the
    merged (out bf16 [B, 1, H, 512], lse fp32 [B, 1, H]) on every rank."""
    if q.dim() != 4 or q.shape[1] != 1:
        raise ValueError("context-parallel decode takes one query token per sequence (s_q = 1)")
    # the collective runs on the current stream: make `stream` current for all three steps
    with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
        out, lse = decode(q, kv_cache, block_table, cache_seqlens, softmax_scale)
        if not dist.is_initialized():
            return out, lse
        out_parts, lse_parts = gather_states(out, lse, group)
        return merge_states(out_parts, lse_parts)
