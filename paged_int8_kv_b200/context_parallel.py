"""Context-parallel decode: one long context spread over several GPUs.

Each rank holds the blocks of a contiguous, chunk-aligned part of every
sequence's context (its own cache, block tables and lengths for that part),
computes that part's chunk partials with kv8_paged_decode_attention_partials,
the ranks all-gather the partials (``torch.distributed``, NCCL over NVLink
on GPUs), and every rank merges all of them with kv8_merge_partials.  The
exchange is (2 + head_dim) fp32 per chunk slot and query head, independent of
the context length; the attention itself runs in the library's kernels.

Context partitioning across devices follows garden.houmin.site
infra/kv-cache-optimize, §4.1.2 KV-Runahead.  This module is plumbing:
shard bounds, table views and the collective; no arithmetic of the method.
"""
from __future__ import annotations

import math

import torch

from . import _binding as B


def shard_bounds(context_len: int, world: int, rank: int,
                 chunk_tokens: int) -> tuple[int, int]:
    """Tokens [begin, end) of a context that rank `rank` of `world` holds:
    the context's chunks of `chunk_tokens` split as evenly as possible into
    contiguous runs, earlier ranks taking the extra chunk."""
    if world <= 0 or not 0 <= rank < world or chunk_tokens <= 0:
        raise ValueError("bad world, rank or chunk_tokens")
    chunks = math.ceil(context_len / chunk_tokens)
    per, extra = divmod(chunks, world)
    c0 = rank * per + min(rank, extra)
    c1 = c0 + per + (1 if rank < extra else 0)
    return min(c0 * chunk_tokens, context_len), min(c1 * chunk_tokens, context_len)


def max_local_len(context_lens, world: int, chunk_tokens: int) -> int:
    """The longest part any rank holds of any context: the bound every rank
    passes as max_context_len, so that their partial layouts match."""
    return max([e - s for n in context_lens for s, e in
                (shard_bounds(int(n), world, r, chunk_tokens)
                 for r in range(world))] + [0])


def local_tables(block_tables, context_lens, world: int, rank: int,
                 chunk_tokens: int, block_size: int = 16):
    """A rank's block tables and lengths for its part of every sequence,
    sliced from global (host) tables: row b lists the blocks of tokens
    [begin_b, end_b).  Returns (tables [B, width], lens [B], bound) where
    bound = max_local_len(...) is the same on every rank and the tables are
    width = ceil(bound / block_size) wide on every rank (padding entries
    are never read); works on numpy arrays or CPU tensors."""
    import numpy as np
    bt = np.asarray(block_tables)
    lens = np.asarray(context_lens)
    spans = [shard_bounds(int(n), world, rank, chunk_tokens) for n in lens]
    nblk = [math.ceil((e - s) / block_size) for s, e in spans]
    bound = max_local_len(lens, world, chunk_tokens)
    width = max(math.ceil(bound / block_size), 1)
    out = np.zeros((bt.shape[0], width), dtype=np.int32)
    for b, (s, e) in enumerate(spans):
        j0 = s // block_size
        out[b, :nblk[b]] = bt[b, j0:j0 + nblk[b]]
    local = np.asarray([e - s for s, e in spans], dtype=np.int32)
    return out, local, bound


def context_parallel_decode(q: torch.Tensor, k_cache: torch.Tensor,
                            v_cache: torch.Tensor, k_scales: torch.Tensor,
                            v_scales: torch.Tensor, local_block_tables: torch.Tensor,
                            local_lens: torch.Tensor, out: torch.Tensor,
                            max_local_len: int, chunk_tokens: int,
                            group=None) -> torch.Tensor:
    """Decode one step of attention over contexts spread across the ranks of
    `group`: this rank's partials, an all-gather, the merge into `out` on
    every rank.  `max_local_len` must be the same bound on every rank."""
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    Bsz, hq, d = q.shape
    nbytes = B.kv8_decode_partials_bytes(Bsz, hq, d, max_local_len, chunk_tokens)
    stride = (nbytes + 255) // 256 * 256
    mine = torch.empty(stride, dtype=torch.uint8, device=q.device)
    B.kv8_paged_decode_attention_partials(
        q, k_cache, v_cache, k_scales, v_scales, local_block_tables,
        local_lens, mine, max_local_len, chunk_tokens)
    allp = gather_partials(mine, world, group)
    return B.kv8_merge_partials(allp, stride, world, out, max_local_len,
                                chunk_tokens)


def gather_partials(mine: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-gather of every rank's partial buffer (the same byte size on every
    rank): rank r's bytes at offset r * mine.numel() of the result, on every
    rank."""
    if world == 1:
        return mine
    import torch.distributed as dist
    allp = torch.empty(world * mine.numel(), dtype=mine.dtype, device=mine.device)
    if mine.is_cuda:
        dist.all_gather_into_tensor(allp, mine, group=group)
    else:  # host ranks (gloo): the list form
        dist.all_gather(list(allp.chunk(world)), mine, group=group)
    return allp
