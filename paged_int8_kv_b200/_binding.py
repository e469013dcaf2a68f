"""ctypes binding of libkv8 (include/kv8.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does
nothing but turn torch tensors into pointers and sizes, pass the current CUDA
stream, and raise ``Kv8Error`` on a non-zero status.  All computation runs in
the CUDA kernels of ``libkv8.so``; there is no Python or CPU fallback, and a
missing or unloadable library raises at import of this module.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkv8.so")

KV8_OK = 0
KV8_ERR_INVALID_ARG = 1
KV8_ERR_UNSUPPORTED = 2
KV8_ERR_WORKSPACE = 3
KV8_ERR_CUDA = 4
KV8_OUT_BF16 = 0
KV8_OUT_F32 = 1
KV8_FORM_AUTO = 0
KV8_FORM_CUDA_CORE = 1
KV8_FORM_MMA_F16PV = 2
KV8_FORM_TCGEN05 = 3
KV8_FORM_MMA_I8 = 4

EXPORTED = (
    "kv8_status_string",
    "kv8_quantize_append",
    "kv8_decode_workspace_bytes",
    "kv8_decode_chunk_tokens",
    "kv8_paged_decode_attention",
    "kv8_split_reduce",
    "kv8_paged_decode_attention_form",
    "kv8_paged_decode_attention_prefix",
    "kv8_paged_extend_attention",
    "kv8_decode_partials_bytes",
    "kv8_paged_decode_attention_partials",
    "kv8_merge_partials",
    "kv8_read_device_status",
    "kv8_paged_decode_attention_noalloc",
    "kv8_paged_decode_attention_append",
    "kv8_int4_quantize_append",
    "kv8_int4_paged_decode_attention",
    "kv8_kivi_append",
    "kv8_kivi_paged_decode_attention",
    "kv8_check_indices",
)

KV8_KIVI_PAGE_BYTES = 2176


class Kv8Error(RuntimeError):
    def __init__(self, func: str, status: int, name: str):
        super().__init__(f"{func} failed: {name} ({status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libkv8.so not found at {LIB_PATH}; build it with "
            "`python -m paged_int8_kv_b200.build` (there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    sz = ctypes.c_size_t
    lib.kv8_status_string.restype = ctypes.c_char_p
    lib.kv8_status_string.argtypes = [i32]
    lib.kv8_quantize_append.restype = i32
    lib.kv8_quantize_append.argtypes = [P, P, P, i64, i32, i32, i32, i64, P, P, P, P, P]
    lib.kv8_decode_workspace_bytes.restype = sz
    lib.kv8_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    lib.kv8_decode_chunk_tokens.restype = i32
    lib.kv8_decode_chunk_tokens.argtypes = [i32, i32, i32]
    lib.kv8_paged_decode_attention.restype = i32
    lib.kv8_paged_decode_attention.argtypes = [
        P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32, f32, i32,
        P, sz, P, i32, P]
    lib.kv8_paged_decode_attention_prefix.restype = i32
    lib.kv8_paged_decode_attention_prefix.argtypes = [
        P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32, P, P,
        i32, i32, i32, f32, i32, P, sz, P, i32, P]
    lib.kv8_paged_extend_attention.restype = i32
    lib.kv8_paged_extend_attention.argtypes = [
        P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32, f32,
        P, i32, P]
    lib.kv8_decode_partials_bytes.restype = sz
    lib.kv8_decode_partials_bytes.argtypes = [i32, i32, i32, i32, i32]
    lib.kv8_paged_decode_attention_partials.restype = i32
    lib.kv8_paged_decode_attention_partials.argtypes = [
        P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32, f32, i32,
        P, sz, P]
    lib.kv8_merge_partials.restype = i32
    lib.kv8_merge_partials.argtypes = [P, sz, i32, i32, i32, i32, i32, i32,
                                       P, i32, P]
    lib.kv8_split_reduce.restype = i32
    lib.kv8_split_reduce.argtypes = [P, sz, P, i32, i32, i32, i32, i32, P, i32, P]
    lib.kv8_paged_decode_attention_form.restype = i32
    lib.kv8_paged_decode_attention_form.argtypes = [
        P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32, f32, i32,
        P, sz, P, i32, i32, P]
    lib.kv8_paged_decode_attention_noalloc.restype = i32
    lib.kv8_paged_decode_attention_noalloc.argtypes = [
        P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32, f32, i32,
        P, i32, P]
    lib.kv8_paged_decode_attention_append.restype = i32
    lib.kv8_paged_decode_attention_append.argtypes = [
        P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32, f32,
        i32, P, sz, P, i32, P]
    lib.kv8_int4_quantize_append.restype = i32
    lib.kv8_int4_quantize_append.argtypes = [P, P, P, i64, i32, i32, i32, i64, P, P, P, P, P]
    lib.kv8_int4_paged_decode_attention.restype = i32
    lib.kv8_int4_paged_decode_attention.argtypes = [
        P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32, f32, i32,
        P, sz, P, i32, P]
    lib.kv8_kivi_append.restype = i32
    lib.kv8_kivi_append.argtypes = [
        P, P, P, P, P, i32, i32, i32, i32, i32, i64, i32, P, P, P]
    lib.kv8_kivi_paged_decode_attention.restype = i32
    lib.kv8_kivi_paged_decode_attention.argtypes = [
        P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32, f32, i32, P, sz,
        P, i32, P]
    lib.kv8_check_indices.restype = i32
    lib.kv8_check_indices.argtypes = [P, P, i32, i32, i64, i32, P, i64, P, P]
    lib.kv8_read_device_status.restype = i32
    lib.kv8_read_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
    return lib


lib = _load()


def _check(func: str, status: int) -> None:
    if status != KV8_OK:
        raise Kv8Error(func, status, lib.kv8_status_string(status).decode())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _p(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    return ctypes.c_void_p(t.data_ptr())


def kv8_status_string(status: int) -> str:
    return lib.kv8_status_string(status).decode()


def kv8_quantize_append(k_new: torch.Tensor, v_new: torch.Tensor,
                        slot_mapping: torch.Tensor, k_cache: torch.Tensor,
                        v_cache: torch.Tensor, k_scales: torch.Tensor,
                        v_scales: torch.Tensor, stream=None) -> None:
    """k_new/v_new bf16 [n, H_kv, D]; slot_mapping int64 [n]; caches int8
    [NB, H_kv, 16, D]; scales fp32 [NB, H_kv, 16] (all on the GPU)."""
    nb, hkv, bs, d = k_cache.shape
    _check("kv8_quantize_append", lib.kv8_quantize_append(
        _p(k_new), _p(v_new), _p(slot_mapping), slot_mapping.shape[0], hkv, d,
        bs, nb, _p(k_cache), _p(v_cache), _p(k_scales), _p(v_scales),
        _stream(stream)))


def kv8_int4_quantize_append(k_new: torch.Tensor, v_new: torch.Tensor,
                             slot_mapping: torch.Tensor, k_cache: torch.Tensor,
                             v_cache: torch.Tensor, k_scales: torch.Tensor,
                             v_scales: torch.Tensor, stream=None) -> None:
    """INT4 cache: k_new/v_new bf16 [n, H_kv, D]; caches uint8
    [NB, H_kv, 16, D/2] (packed excess-8 nibbles); scales fp32 [NB, H_kv, 16]."""
    nb, hkv, bs, dh = k_cache.shape
    _check("kv8_int4_quantize_append", lib.kv8_int4_quantize_append(
        _p(k_new), _p(v_new), _p(slot_mapping), slot_mapping.shape[0], hkv,
        2 * dh, bs, nb, _p(k_cache), _p(v_cache), _p(k_scales), _p(v_scales),
        _stream(stream)))


def kv8_decode_workspace_bytes(batch: int, num_q_heads: int, head_dim: int,
                               max_context_len: int, chunk_tokens: int) -> int:
    return int(lib.kv8_decode_workspace_bytes(batch, num_q_heads, head_dim,
                                              max_context_len, chunk_tokens))


def kv8_decode_chunk_tokens(batch: int, num_kv_heads: int,
                            max_context_len: int) -> int:
    """Suggested chunk_tokens for this device (0: no split)."""
    return int(lib.kv8_decode_chunk_tokens(batch, num_kv_heads, max_context_len))


def _decode_args(q, k_cache, v_cache, k_scales, v_scales, block_tables,
                 context_lens, out, max_context_len, chunk_tokens, workspace,
                 softmax_scale):
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    out_dtype = KV8_OUT_F32 if out.dtype == torch.float32 else KV8_OUT_BF16
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return (_p(q), _p(k_cache), _p(v_cache), _p(k_scales), _p(v_scales),
            _p(block_tables), _p(context_lens), B, hq, hkv, d, bs,
            block_tables.shape[1], nb, int(max_context_len),
            float(softmax_scale), int(chunk_tokens), _p(workspace), ws_bytes,
            _p(out), out_dtype)


def kv8_paged_decode_attention(q: torch.Tensor, k_cache: torch.Tensor,
                               v_cache: torch.Tensor, k_scales: torch.Tensor,
                               v_scales: torch.Tensor,
                               block_tables: torch.Tensor,
                               context_lens: torch.Tensor, out: torch.Tensor,
                               max_context_len: int, chunk_tokens: int = 512,
                               workspace: torch.Tensor | None = None,
                               softmax_scale: float = 0.0,
                               stream=None) -> torch.Tensor:
    """q bf16 [B, H_q, D]; out bf16 or fp32 [B, H_q, D] (written in place)."""
    _check("kv8_paged_decode_attention", lib.kv8_paged_decode_attention(
        *_decode_args(q, k_cache, v_cache, k_scales, v_scales, block_tables,
                      context_lens, out, max_context_len, chunk_tokens,
                      workspace, softmax_scale), _stream(stream)))
    return out


def kv8_paged_decode_attention_form(q: torch.Tensor, k_cache: torch.Tensor,
                                    v_cache: torch.Tensor,
                                    k_scales: torch.Tensor,
                                    v_scales: torch.Tensor,
                                    block_tables: torch.Tensor,
                                    context_lens: torch.Tensor,
                                    out: torch.Tensor, max_context_len: int,
                                    chunk_tokens: int = 512,
                                    workspace: torch.Tensor | None = None,
                                    softmax_scale: float = 0.0,
                                    form: int = KV8_FORM_AUTO,
                                    stream=None) -> torch.Tensor:
    """kv8_paged_decode_attention with the decode form given for this call."""
    _check("kv8_paged_decode_attention_form",
           lib.kv8_paged_decode_attention_form(
               *_decode_args(q, k_cache, v_cache, k_scales, v_scales,
                             block_tables, context_lens, out, max_context_len,
                             chunk_tokens, workspace, softmax_scale),
               int(form), _stream(stream)))
    return out


def kv8_int4_paged_decode_attention(q: torch.Tensor, k_cache: torch.Tensor,
                                    v_cache: torch.Tensor,
                                    k_scales: torch.Tensor,
                                    v_scales: torch.Tensor,
                                    block_tables: torch.Tensor,
                                    context_lens: torch.Tensor,
                                    out: torch.Tensor, max_context_len: int,
                                    chunk_tokens: int = 512,
                                    workspace: torch.Tensor | None = None,
                                    softmax_scale: float = 0.0,
                                    stream=None) -> torch.Tensor:
    """Decode attention over the INT4 cache (uint8 [NB, H_kv, 16, D/2])."""
    _check("kv8_int4_paged_decode_attention",
           lib.kv8_int4_paged_decode_attention(
               *_decode_args(q, k_cache, v_cache, k_scales, v_scales,
                             block_tables, context_lens, out, max_context_len,
                             chunk_tokens, workspace, softmax_scale),
               _stream(stream)))
    return out


def kv8_check_indices(block_tables: torch.Tensor | None,
                      context_lens: torch.Tensor | None, max_context_len: int,
                      num_blocks: int, slot_mapping: torch.Tensor | None = None,
                      stream=None) -> tuple[int, int, int]:
    """Debug check of the trusted indices: returns (context lengths out of
    [0, max_context_len], block-table entries a decode would read outside
    [0, num_blocks), slots at or past num_blocks * 16), after synchronising
    the stream."""
    given = [t for t in (block_tables, context_lens, slot_mapping) if t is not None]
    if not given:
        raise ValueError("kv8_check_indices: nothing to check")
    dev = given[0].device
    counts = torch.zeros(3, dtype=torch.int32, device=dev)
    batch = 0 if context_lens is None else context_lens.shape[0]
    mbs = 1 if block_tables is None else block_tables.shape[1]
    n = 0 if slot_mapping is None else slot_mapping.shape[0]
    st = _stream(stream)
    _check("kv8_check_indices", lib.kv8_check_indices(
        _p(block_tables), _p(context_lens), batch, mbs, int(num_blocks),
        int(max_context_len), _p(slot_mapping), n, _p(counts), st))
    if stream is None:
        torch.cuda.current_stream(dev).synchronize()
    else:
        stream.synchronize()
    return tuple(int(x) for x in counts.cpu().tolist())


def kv8_kivi_append(k_new: torch.Tensor, v_new: torch.Tensor,
                    cu_new: torch.Tensor, context_lens: torch.Tensor,
                    block_tables: torch.Tensor, kivi_cache: torch.Tensor,
                    kivi_tail: torch.Tensor, max_new_tokens: int,
                    stream=None) -> None:
    """Append rows to the KIVI cache: k_new/v_new bf16 [N, H_kv, D], cu_new
    int32 [B + 1], context_lens int32 [B] (after the append); kivi_cache
    uint8 [NB, H_kv, KV8_KIVI_PAGE_BYTES]; kivi_tail bf16
    [B, H_kv, 2, 16, D]."""
    nb, hkv, _ = kivi_cache.shape
    B = context_lens.shape[0]
    _check("kv8_kivi_append", lib.kv8_kivi_append(
        _p(k_new), _p(v_new), _p(cu_new), _p(context_lens), _p(block_tables),
        B, hkv, kivi_tail.shape[-1], kivi_tail.shape[-2], block_tables.shape[1],
        nb, int(max_new_tokens), _p(kivi_cache), _p(kivi_tail),
        _stream(stream)))


def kv8_kivi_paged_decode_attention(q: torch.Tensor, kivi_cache: torch.Tensor,
                                    kivi_tail: torch.Tensor,
                                    block_tables: torch.Tensor,
                                    context_lens: torch.Tensor,
                                    out: torch.Tensor, max_context_len: int,
                                    chunk_tokens: int = 512,
                                    workspace: torch.Tensor | None = None,
                                    softmax_scale: float = 0.0,
                                    stream=None) -> torch.Tensor:
    """Decode attention over the KIVI cache; q bf16 [B, H_q, D], out bf16
    or fp32 [B, H_q, D] (written in place)."""
    B, hq, d = q.shape
    nb, hkv, _ = kivi_cache.shape
    out_dtype = KV8_OUT_F32 if out.dtype == torch.float32 else KV8_OUT_BF16
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("kv8_kivi_paged_decode_attention",
           lib.kv8_kivi_paged_decode_attention(
               _p(q), _p(kivi_cache), _p(kivi_tail), _p(block_tables),
               _p(context_lens), B, hq, hkv, d, kivi_tail.shape[-2],
               block_tables.shape[1], nb, int(max_context_len),
               float(softmax_scale), int(chunk_tokens), _p(workspace),
               ws_bytes, _p(out), out_dtype, _stream(stream)))
    return out


def kv8_paged_decode_attention_append(q: torch.Tensor, k_new: torch.Tensor,
                                      v_new: torch.Tensor, k_cache: torch.Tensor,
                                      v_cache: torch.Tensor,
                                      k_scales: torch.Tensor,
                                      v_scales: torch.Tensor,
                                      block_tables: torch.Tensor,
                                      context_lens: torch.Tensor,
                                      out: torch.Tensor, max_context_len: int,
                                      chunk_tokens: int = 512,
                                      workspace: torch.Tensor | None = None,
                                      softmax_scale: float = 0.0,
                                      stream=None) -> torch.Tensor:
    """One decode step in one launch: k_new / v_new bf16 [B, H_kv, D] (token
    b at position context_lens[b] - 1) quantised into the cache, then the
    decode attention; out written in place."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    out_dtype = KV8_OUT_F32 if out.dtype == torch.float32 else KV8_OUT_BF16
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("kv8_paged_decode_attention_append",
           lib.kv8_paged_decode_attention_append(
               _p(q), _p(k_new), _p(v_new), _p(k_cache), _p(v_cache),
               _p(k_scales), _p(v_scales), _p(block_tables), _p(context_lens),
               B, hq, hkv, d, bs, block_tables.shape[1], nb,
               int(max_context_len), float(softmax_scale), int(chunk_tokens),
               _p(workspace), ws_bytes, _p(out), out_dtype, _stream(stream)))
    return out


def kv8_paged_decode_attention_prefix(q: torch.Tensor, k_cache: torch.Tensor,
                                      v_cache: torch.Tensor,
                                      k_scales: torch.Tensor,
                                      v_scales: torch.Tensor,
                                      block_tables: torch.Tensor,
                                      context_lens: torch.Tensor,
                                      out: torch.Tensor, max_context_len: int,
                                      prefix_group: torch.Tensor,
                                      prefix_lens: torch.Tensor,
                                      max_group_size: int, max_prefix_len: int,
                                      chunk_tokens: int = 512,
                                      workspace: torch.Tensor | None = None,
                                      softmax_scale: float = 0.0,
                                      stream=None) -> torch.Tensor:
    """Decode with shared prefixes: prefix_group int32 [B] (-1 = none),
    prefix_lens int32 [num_groups] (both on the GPU)."""
    a = _decode_args(q, k_cache, v_cache, k_scales, v_scales, block_tables,
                     context_lens, out, max_context_len, chunk_tokens,
                     workspace, softmax_scale)
    _check("kv8_paged_decode_attention_prefix",
           lib.kv8_paged_decode_attention_prefix(
               *a[:15], _p(prefix_group), _p(prefix_lens),
               int(prefix_lens.shape[0]), int(max_group_size),
               int(max_prefix_len), *a[15:], _stream(stream)))
    return out


def kv8_paged_extend_attention(q: torch.Tensor, k_cache: torch.Tensor,
                               v_cache: torch.Tensor, k_scales: torch.Tensor,
                               v_scales: torch.Tensor,
                               block_tables: torch.Tensor,
                               context_lens: torch.Tensor,
                               q_start: torch.Tensor, out: torch.Tensor,
                               max_q_len: int, softmax_scale: float = 0.0,
                               stream=None) -> torch.Tensor:
    """q bf16 [rows, H_q, D] (new rows of every sequence, packed);
    q_start int32 [B+1]; out bf16 or fp32 like q (written in place)."""
    nq, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    out_dtype = KV8_OUT_F32 if out.dtype == torch.float32 else KV8_OUT_BF16
    _check("kv8_paged_extend_attention", lib.kv8_paged_extend_attention(
        _p(q), _p(k_cache), _p(v_cache), _p(k_scales), _p(v_scales),
        _p(block_tables), _p(context_lens), _p(q_start),
        int(context_lens.shape[0]), hq, hkv, d, bs, block_tables.shape[1], nb,
        int(max_q_len), float(softmax_scale), _p(out), out_dtype,
        _stream(stream)))
    return out


def kv8_paged_decode_attention_noalloc(q: torch.Tensor, k_cache: torch.Tensor,
                                       v_cache: torch.Tensor,
                                       k_scales: torch.Tensor,
                                       v_scales: torch.Tensor,
                                       block_tables: torch.Tensor,
                                       context_lens: torch.Tensor,
                                       out: torch.Tensor, max_context_len: int,
                                       chunk_tokens: int = 512,
                                       softmax_scale: float = 0.0,
                                       stream=None) -> torch.Tensor:
    """Like kv8_paged_decode_attention, for callers that cannot allocate:
    the split partials use the library's fixed per-device scratch array."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    out_dtype = KV8_OUT_F32 if out.dtype == torch.float32 else KV8_OUT_BF16
    _check("kv8_paged_decode_attention_noalloc",
           lib.kv8_paged_decode_attention_noalloc(
               _p(q), _p(k_cache), _p(v_cache), _p(k_scales), _p(v_scales),
               _p(block_tables), _p(context_lens), B, hq, hkv, d, bs,
               block_tables.shape[1], nb, int(max_context_len),
               float(softmax_scale), int(chunk_tokens), _p(out), out_dtype,
               _stream(stream)))
    return out


def kv8_decode_partials_bytes(batch: int, num_q_heads: int, head_dim: int,
                              max_context_len: int, chunk_tokens: int) -> int:
    return int(lib.kv8_decode_partials_bytes(batch, num_q_heads, head_dim,
                                             max_context_len, chunk_tokens))


def kv8_paged_decode_attention_partials(q: torch.Tensor, k_cache: torch.Tensor,
                                        v_cache: torch.Tensor,
                                        k_scales: torch.Tensor,
                                        v_scales: torch.Tensor,
                                        block_tables: torch.Tensor,
                                        context_lens: torch.Tensor,
                                        partials: torch.Tensor,
                                        max_context_len: int,
                                        chunk_tokens: int,
                                        softmax_scale: float = 0.0,
                                        stream=None) -> torch.Tensor:
    """One rank's chunk partials of a context-parallel decode (uint8 buffer
    of kv8_decode_partials_bytes bytes, written in place)."""
    B, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    _check("kv8_paged_decode_attention_partials",
           lib.kv8_paged_decode_attention_partials(
               _p(q), _p(k_cache), _p(v_cache), _p(k_scales), _p(v_scales),
               _p(block_tables), _p(context_lens), B, hq, hkv, d, bs,
               block_tables.shape[1], nb, int(max_context_len),
               float(softmax_scale), int(chunk_tokens), _p(partials),
               partials.numel() * partials.element_size(), _stream(stream)))
    return partials


def kv8_merge_partials(partials: torch.Tensor, rank_stride: int, ranks: int,
                       out: torch.Tensor, max_context_len: int,
                       chunk_tokens: int, stream=None) -> torch.Tensor:
    """Merge `ranks` partial buffers (rank r at byte r * rank_stride of
    `partials`) into out [B, H_q, D] (bf16 or fp32, written in place)."""
    B, hq, d = out.shape
    out_dtype = KV8_OUT_F32 if out.dtype == torch.float32 else KV8_OUT_BF16
    _check("kv8_merge_partials", lib.kv8_merge_partials(
        _p(partials), int(rank_stride), int(ranks), B, hq, d,
        int(max_context_len), int(chunk_tokens), _p(out), out_dtype,
        _stream(stream)))
    return out


def kv8_split_reduce(workspace: torch.Tensor, context_lens: torch.Tensor,
                     out: torch.Tensor, max_context_len: int,
                     chunk_tokens: int, stream=None) -> torch.Tensor:
    B, hq, d = out.shape
    out_dtype = KV8_OUT_F32 if out.dtype == torch.float32 else KV8_OUT_BF16
    _check("kv8_split_reduce", lib.kv8_split_reduce(
        _p(workspace), workspace.numel() * workspace.element_size(),
        _p(context_lens), B, hq, d, int(max_context_len), int(chunk_tokens),
        _p(out), out_dtype, _stream(stream)))
    return out


def kv8_read_device_status(clear: bool = True) -> int:
    v = ctypes.c_uint32(0)
    _check("kv8_read_device_status", lib.kv8_read_device_status(ctypes.byref(v), int(clear)))
    return int(v.value)


def default_softmax_scale(head_dim: int = 128) -> float:
    return 1.0 / math.sqrt(head_dim)
