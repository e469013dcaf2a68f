"""Device-memory owner for one layer's paged INT8 KV cache.

``PagedKV8Cache`` allocates the four cache tensors (codes and scales for K
and V, layout as in include/kv8.h) and a reusable split-K workspace with
PyTorch, and forwards to the C entry points.  It is plumbing only: every
number it produces comes from the CUDA kernels.

Debug mode: with the environment variable ``KV8_DEBUG`` set (to anything but
``0``), every append, decode and step first runs ``kv8_check_indices`` on
the indices it is given (slots; block tables and context lengths) and raises
``ValueError`` instead of launching when any is out of range.  The calls
themselves trust those indices.
"""
from __future__ import annotations

import os

import torch

from . import _binding as B


def debug_checks_enabled() -> bool:
    return os.environ.get("KV8_DEBUG", "") not in ("", "0")


def check_indices(num_blocks: int, block_tables=None, context_lens=None,
                  max_context_len: int = 0, slot_mapping=None, stream=None) -> None:
    """Raise ValueError if kv8_check_indices finds an index out of range."""
    bad = B.kv8_check_indices(block_tables, context_lens, max_context_len,
                              num_blocks, slot_mapping=slot_mapping, stream=stream)
    if any(bad):
        raise ValueError(
            f"KV8_DEBUG: {bad[0]} context lengths outside [0, {max_context_len}], "
            f"{bad[1]} block-table entries outside [0, {num_blocks}), "
            f"{bad[2]} slots past the cache's {num_blocks * 16}")


class PagedKV8Cache:
    def __init__(self, num_blocks: int, num_kv_heads: int, head_dim: int = 128,
                 block_size: int = 16, device: str | torch.device = "cuda",
                 poison: bool = True):
        self.num_blocks = int(num_blocks)
        self.num_kv_heads = int(num_kv_heads)
        self.head_dim = int(head_dim)
        self.block_size = int(block_size)
        self.device = torch.device(device)
        shape = (self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim)
        sshape = shape[:3]
        self.k_cache = torch.empty(shape, dtype=torch.int8, device=self.device)
        self.v_cache = torch.empty(shape, dtype=torch.int8, device=self.device)
        self.k_scales = torch.empty(sshape, dtype=torch.float32, device=self.device)
        self.v_scales = torch.empty(sshape, dtype=torch.float32, device=self.device)
        if poison:
            self.poison()
        self._ws = None

    def poison(self) -> None:
        """Unwritten slots read as code 127 with a NaN scale."""
        self.k_cache.fill_(127)
        self.v_cache.fill_(127)
        self.k_scales.fill_(float("nan"))
        self.v_scales.fill_(float("nan"))

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size()
                   for t in (self.k_cache, self.v_cache, self.k_scales, self.v_scales))

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor,
               slot_mapping: torch.Tensor, stream=None) -> None:
        if debug_checks_enabled():
            check_indices(self.num_blocks, slot_mapping=slot_mapping, stream=stream)
        B.kv8_quantize_append(k_new, v_new, slot_mapping, self.k_cache,
                              self.v_cache, self.k_scales, self.v_scales,
                              stream=stream)

    def workspace(self, batch: int, num_q_heads: int, max_context_len: int,
                  chunk_tokens: int) -> torch.Tensor | None:
        need = B.kv8_decode_workspace_bytes(batch, num_q_heads, self.head_dim,
                                            max_context_len, chunk_tokens)
        if need == 0:
            return None
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def decode(self, q: torch.Tensor, block_tables: torch.Tensor,
               context_lens: torch.Tensor, max_context_len: int,
               chunk_tokens: int = 512, out: torch.Tensor | None = None,
               out_dtype: torch.dtype = torch.bfloat16,
               softmax_scale: float = 0.0, form: int = B.KV8_FORM_AUTO,
               stream=None) -> torch.Tensor:
        """One decode step over this cache; ``form`` picks the decode form
        for this call (KV8_FORM_AUTO: the library's default)."""
        if debug_checks_enabled():
            check_indices(self.num_blocks, block_tables, context_lens,
                          max_context_len, stream=stream)
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        ws = self.workspace(q.shape[0], q.shape[1], max_context_len, chunk_tokens)
        return B.kv8_paged_decode_attention_form(
            q, self.k_cache, self.v_cache, self.k_scales, self.v_scales,
            block_tables, context_lens, out, max_context_len,
            chunk_tokens=chunk_tokens, workspace=ws,
            softmax_scale=softmax_scale, form=form, stream=stream)

    def step(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
             block_tables: torch.Tensor, context_lens: torch.Tensor,
             max_context_len: int, chunk_tokens: int = 512,
             out: torch.Tensor | None = None,
             out_dtype: torch.dtype = torch.bfloat16,
             softmax_scale: float = 0.0, stream=None) -> torch.Tensor:
        """One decode step in one launch: sequence b's new K/V (bf16
        [B, H_kv, D]) join the cache at position context_lens[b] - 1, then
        every query head attends over the whole context."""
        if debug_checks_enabled():
            check_indices(self.num_blocks, block_tables, context_lens,
                          max_context_len, stream=stream)
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        ws = self.workspace(q.shape[0], q.shape[1], max_context_len, chunk_tokens)
        return B.kv8_paged_decode_attention_append(
            q, k_new, v_new, self.k_cache, self.v_cache, self.k_scales,
            self.v_scales, block_tables, context_lens, out, max_context_len,
            chunk_tokens=chunk_tokens, workspace=ws,
            softmax_scale=softmax_scale, stream=stream)


class PagedKiviCache:
    """Device memory of one layer's KIVI cache: the page records
    (uint8 [num_blocks, H_kv, KV8_KIVI_PAGE_BYTES]) and the bf16 tail of each
    batch row's partial page ([batch, H_kv, 2, 16, 128]); forwards to
    kv8_kivi_append and kv8_kivi_paged_decode_attention."""

    def __init__(self, num_blocks: int, num_kv_heads: int, batch: int,
                 head_dim: int = 128, block_size: int = 16,
                 device: str | torch.device = "cuda"):
        self.num_blocks = int(num_blocks)
        self.num_kv_heads = int(num_kv_heads)
        self.batch = int(batch)
        self.head_dim = int(head_dim)
        self.block_size = int(block_size)
        self.device = torch.device(device)
        self.records = torch.zeros((self.num_blocks, self.num_kv_heads,
                                    B.KV8_KIVI_PAGE_BYTES), dtype=torch.uint8,
                                   device=self.device)
        self.tail = torch.zeros((self.batch, self.num_kv_heads, 2,
                                 self.block_size, self.head_dim),
                                dtype=torch.bfloat16, device=self.device)
        self._ws = None

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor,
               cu_new: torch.Tensor, context_lens: torch.Tensor,
               block_tables: torch.Tensor, max_new_tokens: int,
               stream=None) -> None:
        """Batch row b's new rows are k_new/v_new[cu_new[b] : cu_new[b+1]],
        at its last positions (context_lens counts them)."""
        if debug_checks_enabled():
            check_indices(self.num_blocks, block_tables, context_lens,
                          block_tables.shape[1] * self.block_size, stream=stream)
        B.kv8_kivi_append(k_new, v_new, cu_new, context_lens, block_tables,
                          self.records, self.tail, max_new_tokens, stream=stream)

    def workspace(self, batch: int, num_q_heads: int, max_context_len: int,
                  chunk_tokens: int) -> torch.Tensor | None:
        need = B.kv8_decode_workspace_bytes(batch, num_q_heads, self.head_dim,
                                            max_context_len, chunk_tokens)
        if need == 0:
            return None
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def decode(self, q: torch.Tensor, block_tables: torch.Tensor,
               context_lens: torch.Tensor, max_context_len: int,
               chunk_tokens: int = 512, out: torch.Tensor | None = None,
               out_dtype: torch.dtype = torch.bfloat16,
               softmax_scale: float = 0.0, stream=None) -> torch.Tensor:
        if debug_checks_enabled():
            check_indices(self.num_blocks, block_tables, context_lens,
                          max_context_len, stream=stream)
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        ws = self.workspace(q.shape[0], q.shape[1], max_context_len, chunk_tokens)
        return B.kv8_kivi_paged_decode_attention(
            q, self.records, self.tail, block_tables, context_lens, out,
            max_context_len, chunk_tokens=chunk_tokens, workspace=ws,
            softmax_scale=softmax_scale, stream=stream)


def fill_from_host(cache: PagedKV8Cache, segments, stream=None) -> int:
    """Copy host (k, v, slot_mapping) segments to the GPU and append them.

    ``segments`` yields numpy arrays: k and v as bf16 bit patterns (uint16)
    [n, H_kv, D] and slot_mapping int64 [n].  Returns the number of tokens
    appended.  Each segment is staged through pinned memory.
    """
    total = 0
    for k, v, slots in segments:
        n = int(slots.shape[0])
        if n == 0:
            continue
        kt = torch.from_numpy(k).view(torch.bfloat16).pin_memory().to(cache.device, non_blocking=True)
        vt = torch.from_numpy(v).view(torch.bfloat16).pin_memory().to(cache.device, non_blocking=True)
        st = torch.from_numpy(slots).pin_memory().to(cache.device, non_blocking=True)
        cache.append(kt, vt, st, stream=stream)
        total += n
    return total
