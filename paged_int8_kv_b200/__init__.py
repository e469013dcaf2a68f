"""paged_int8_kv_b200 -- paged INT8 KV-cache decode attention for B200.

The computation lives in ``libkv8.so`` (CUDA for sm_100a, C ABI declared in
``include/kv8.h``).  This package only loads that library and marshals
arguments; see ``_binding`` for the functions, which carry the C names.

    from paged_int8_kv_b200 import kv8_quantize_append, kv8_paged_decode_attention

The library is loaded on first use of any of these names (so that
``paged_int8_kv_b200.build`` can run before it exists); if it is missing or
cannot be loaded, that first use raises ImportError.  There is no fallback.
"""
import importlib

_BINDING_NAMES = {
    "EXPORTED", "KV8_ERR_CUDA", "KV8_ERR_INVALID_ARG", "KV8_ERR_UNSUPPORTED",
    "KV8_ERR_WORKSPACE", "KV8_FORM_AUTO", "KV8_FORM_CUDA_CORE",
    "KV8_FORM_MMA_F16PV", "KV8_FORM_MMA_I8", "KV8_FORM_TCGEN05", "KV8_OK", "KV8_OUT_BF16",
    "KV8_OUT_F32", "LIB_PATH",
    "Kv8Error", "default_softmax_scale", "kv8_decode_chunk_tokens",
    "kv8_decode_workspace_bytes",
    "kv8_paged_decode_attention", "kv8_paged_decode_attention_form",
    "kv8_paged_decode_attention_prefix", "kv8_paged_extend_attention",
    "kv8_decode_partials_bytes", "kv8_paged_decode_attention_partials",
    "kv8_merge_partials",
    "kv8_paged_decode_attention_noalloc", "kv8_paged_decode_attention_append",
    "kv8_quantize_append", "kv8_int4_quantize_append",
    "kv8_int4_paged_decode_attention", "kv8_kivi_append",
    "kv8_kivi_paged_decode_attention", "KV8_KIVI_PAGE_BYTES",
    "kv8_check_indices",
    "kv8_read_device_status", "kv8_split_reduce",
    "kv8_status_string",
}
_RUNTIME_NAMES = {"PagedKV8Cache", "PagedKiviCache", "fill_from_host"}
_BLOCK_NAMES = {"BlockAllocator", "OutOfBlocks"}

__all__ = sorted(_BINDING_NAMES | _RUNTIME_NAMES | _BLOCK_NAMES)


def __getattr__(name):
    if name in _BINDING_NAMES:
        return getattr(importlib.import_module("._binding", __name__), name)
    if name in _RUNTIME_NAMES:
        return getattr(importlib.import_module(".runtime", __name__), name)
    if name in _BLOCK_NAMES:
        return getattr(importlib.import_module(".blocks", __name__), name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
