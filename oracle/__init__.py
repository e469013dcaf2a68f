"""CPU oracle for paged INT8 KV decode attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product path (the CUDA
library under ``paged_int8_kv_b200``) never loads it, and the two share no
code: this module wraps ``kv8_oracle.c`` (plain C, single threaded) with
ctypes and adds nothing but argument marshalling.

What each function computes, and the passage it follows, is stated in
``kv8_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kv8_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkv8_oracle.so")

ORACLE_OK = 0
ORACLE_BAD_ARG = 1
ORACLE_NONFINITE = 2
ORACLE_NOMEM = 3

_lib = None


def build(force: bool = False) -> str:
    """Compile kv8_oracle.c into libkv8_oracle.so with gcc (no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp"
    cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    lib.oracle_quantize_append.restype = ctypes.c_int
    lib.oracle_quantize_append.argtypes = [P, P, i64, i32, i32, i32, i64, P, P]
    lib.oracle_decode_attention.restype = ctypes.c_int
    lib.oracle_decode_attention.argtypes = [
        P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, f64, P, i64, P]
    lib.oracle_extend_attention.restype = ctypes.c_int
    lib.oracle_extend_attention.argtypes = [
        P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, f64, P]
    lib.oracle_quantize_append_int4.restype = ctypes.c_int
    lib.oracle_quantize_append_int4.argtypes = [P, P, i64, i32, i32, i32, i64, P, P]
    lib.oracle_decode_attention_int4.restype = ctypes.c_int
    lib.oracle_decode_attention_int4.argtypes = [
        P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, f64, P]
    lib.oracle_kivi_append.restype = ctypes.c_int
    lib.oracle_kivi_append.argtypes = [
        P, P, P, P, P, i32, i32, i32, i32, i32, i64, P, P, P, P, P, P, P]
    lib.oracle_kivi_decode_attention.restype = ctypes.c_int
    lib.oracle_kivi_decode_attention.argtypes = [
        P, P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, f64, P]
    lib.oracle_kv_cache_bytes.restype = f64
    lib.oracle_kv_cache_bytes.argtypes = [i64] * 7
    lib.oracle_kv8_scale_bytes.restype = f64
    lib.oracle_kv8_scale_bytes.argtypes = [i64] * 4
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, what: str):
    if rc != ORACLE_OK:
        raise ValueError(f"{what}: oracle status {rc}")


def quantize_append(x_bf16: np.ndarray, slot_mapping: np.ndarray,
                    cache: np.ndarray, scales: np.ndarray) -> None:
    """Quantise x (uint16 bf16 bits, [n_tokens, H_kv, D]) into cache/scales in place.

    cache: int8 [num_blocks, H_kv, block_size, D]; scales: float32
    [num_blocks, H_kv, block_size].  Both must be C-contiguous.
    """
    lib = _load()
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    assert cache.dtype == np.int8 and cache.flags.c_contiguous
    assert scales.dtype == np.float32 and scales.flags.c_contiguous
    nb, hkv, bs, d = cache.shape
    assert x.shape[1:] == (hkv, d) and sm.shape == (x.shape[0],)
    assert scales.shape == (nb, hkv, bs)
    rc = lib.oracle_quantize_append(_ptr(x), _ptr(sm), x.shape[0], hkv, d, bs,
                                    nb, _ptr(cache), _ptr(scales))
    _check(rc, "oracle_quantize_append")


def decode_attention(q_bf16: np.ndarray, k_cache: np.ndarray,
                     v_cache: np.ndarray, k_scales: np.ndarray,
                     v_scales: np.ndarray, block_tables: np.ndarray,
                     context_lens: np.ndarray, softmax_scale: float = 0.0,
                     pairs=None) -> np.ndarray:
    """fp64 decode attention over the dequantised paged cache.

    q_bf16: uint16 [B, H_q, D].  Returns float64 [B, H_q, D], or
    [len(pairs), D] when ``pairs`` (a list of (b, h)) is given.
    """
    lib = _load()
    q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    for a in (k_cache, v_cache):
        assert a.dtype == np.int8 and a.flags.c_contiguous
    for a in (k_scales, v_scales):
        assert a.dtype == np.float32 and a.flags.c_contiguous
    B, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    assert d2 == d and v_cache.shape == k_cache.shape
    assert bt.shape[0] == B and cl.shape == (B,)
    if pairs is None:
        out = np.zeros((B, hq, d), dtype=np.float64)
        pp, npairs = None, 0
    else:
        pa = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        npairs = pa.shape[0]
        out = np.zeros((npairs, d), dtype=np.float64)
        pp = _ptr(pa)
    rc = lib.oracle_decode_attention(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scales), _ptr(v_scales),
        _ptr(bt), _ptr(cl), B, hq, hkv, d, bs, bt.shape[1], nb,
        float(softmax_scale), pp, npairs, _ptr(out))
    _check(rc, "oracle_decode_attention")
    return out


def extend_attention(q_bf16: np.ndarray, k_cache: np.ndarray,
                     v_cache: np.ndarray, k_scales: np.ndarray,
                     v_scales: np.ndarray, block_tables: np.ndarray,
                     context_lens: np.ndarray, q_start: np.ndarray,
                     softmax_scale: float = 0.0) -> np.ndarray:
    """fp64 causal extend (prefill) attention over the dequantised cache.

    q_bf16: uint16 [q_start[-1], H_q, D], the new query rows of every
    sequence packed in order; sequence b's rows are its last
    q_start[b+1]-q_start[b] cached positions.  Returns float64 of q's shape.
    """
    lib = _load()
    q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    qs = np.ascontiguousarray(q_start, dtype=np.int32)
    for a in (k_cache, v_cache):
        assert a.dtype == np.int8 and a.flags.c_contiguous
    for a in (k_scales, v_scales):
        assert a.dtype == np.float32 and a.flags.c_contiguous
    nq, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    B = cl.shape[0]
    assert d2 == d and qs.shape == (B + 1,) and int(qs[-1]) == nq
    out = np.zeros((nq, hq, d), dtype=np.float64)
    rc = lib.oracle_extend_attention(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scales), _ptr(v_scales),
        _ptr(bt), _ptr(cl), _ptr(qs), B, hq, hkv, d, bs, bt.shape[1], nb,
        float(softmax_scale), _ptr(out))
    _check(rc, "oracle_extend_attention")
    return out


def quantize_append_int4(x_bf16: np.ndarray, slot_mapping: np.ndarray,
                         cache: np.ndarray, scales: np.ndarray) -> None:
    """INT4 variant: quantise x (uint16 bf16 bits, [n, H_kv, D]) into cache
    (uint8 [NB, H_kv, BS, D/2], excess-8 nibbles) and scales (float32
    [NB, H_kv, BS]) in place."""
    lib = _load()
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    assert cache.dtype == np.uint8 and cache.flags.c_contiguous
    assert scales.dtype == np.float32 and scales.flags.c_contiguous
    nb, hkv, bs, dh = cache.shape
    assert x.shape[1:] == (hkv, 2 * dh) and sm.shape == (x.shape[0],)
    rc = lib.oracle_quantize_append_int4(_ptr(x), _ptr(sm), x.shape[0], hkv,
                                         2 * dh, bs, nb, _ptr(cache), _ptr(scales))
    _check(rc, "oracle_quantize_append_int4")


def decode_attention_int4(q_bf16: np.ndarray, k_cache: np.ndarray,
                          v_cache: np.ndarray, k_scales: np.ndarray,
                          v_scales: np.ndarray, block_tables: np.ndarray,
                          context_lens: np.ndarray,
                          softmax_scale: float = 0.0) -> np.ndarray:
    """fp64 decode attention over the dequantised INT4 cache; [B, H_q, D]."""
    lib = _load()
    q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, hq, d = q.shape
    nb, hkv, bs, dh = k_cache.shape
    assert 2 * dh == d and v_cache.shape == k_cache.shape
    out = np.zeros((B, hq, d), dtype=np.float64)
    rc = lib.oracle_decode_attention_int4(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scales), _ptr(v_scales),
        _ptr(bt), _ptr(cl), B, hq, hkv, d, bs, bt.shape[1], nb,
        float(softmax_scale), _ptr(out))
    _check(rc, "oracle_decode_attention_int4")
    return out


class KiviCache:
    """The oracle's KIVI cache in plain layouts (one code per byte):

    k_codes, v_codes uint8 [NB, H_kv, BS, D]; k_scale, k_zero float32
    [NB, H_kv, D] (per channel); v_scale, v_zero float32 [NB, H_kv, BS]
    (per token); tail uint16 bf16 bits [B, H_kv, 2, BS, D] (the K and V rows
    of each sequence's page that is not yet full).  Fields start as
    `fill_code` / NaN / 0xFFFF so that a slot the oracle never writes shows.
    """

    def __init__(self, num_blocks, num_kv_heads, batch, block_size=16,
                 head_dim=128, fill_code=0xFF):
        nb, h, bs, d = num_blocks, num_kv_heads, block_size, head_dim
        self.k_codes = np.full((nb, h, bs, d), fill_code, np.uint8)
        self.v_codes = np.full((nb, h, bs, d), fill_code, np.uint8)
        self.k_scale = np.full((nb, h, d), np.nan, np.float32)
        self.k_zero = np.full((nb, h, d), np.nan, np.float32)
        self.v_scale = np.full((nb, h, bs), np.nan, np.float32)
        self.v_zero = np.full((nb, h, bs), np.nan, np.float32)
        self.tail = np.full((batch, h, 2, bs, d), 0xFFFF, np.uint16)

    def fields(self):
        return (self.k_codes, self.k_scale, self.k_zero, self.v_codes,
                self.v_scale, self.v_zero)


def kivi_append(cache: KiviCache, k_new: np.ndarray, v_new: np.ndarray,
                cu_new: np.ndarray, context_lens: np.ndarray,
                block_tables: np.ndarray) -> None:
    """Append sequence b's rows k_new/v_new[cu_new[b]:cu_new[b+1]] (uint16
    bf16 bits, [N, H_kv, D]) at its last positions (context_lens counts
    them), quantising every page they complete; in place."""
    lib = _load()
    kn = np.ascontiguousarray(k_new, dtype=np.uint16)
    vn = np.ascontiguousarray(v_new, dtype=np.uint16)
    cu = np.ascontiguousarray(cu_new, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    nb, hkv, bs, d = cache.k_codes.shape
    B = cl.shape[0]
    assert cu.shape == (B + 1,) and kn.shape == vn.shape
    assert kn.shape[0] == int(cu[-1]) and kn.shape[1:] == (hkv, d)
    assert bt.shape[0] == B and cache.tail.shape == (B, hkv, 2, bs, d)
    rc = lib.oracle_kivi_append(
        _ptr(kn), _ptr(vn), _ptr(cu), _ptr(cl), _ptr(bt), B, hkv, d, bs,
        bt.shape[1], nb, *[_ptr(a) for a in cache.fields()], _ptr(cache.tail))
    _check(rc, "oracle_kivi_append")


def kivi_decode_attention(q_bf16: np.ndarray, cache: KiviCache,
                          block_tables: np.ndarray, context_lens: np.ndarray,
                          softmax_scale: float = 0.0) -> np.ndarray:
    """fp64 decode attention over the KIVI cache (full pages dequantised,
    the partial page's rows from the tail); [B, H_q, D]."""
    lib = _load()
    q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, hq, d = q.shape
    nb, hkv, bs, d2 = cache.k_codes.shape
    assert d2 == d and bt.shape[0] == B and cl.shape == (B,)
    out = np.zeros((B, hq, d), dtype=np.float64)
    rc = lib.oracle_kivi_decode_attention(
        _ptr(q), *[_ptr(a) for a in cache.fields()], _ptr(cache.tail),
        _ptr(bt), _ptr(cl), B, hq, hkv, d, bs, bt.shape[1], nb,
        float(softmax_scale), _ptr(out))
    _check(rc, "oracle_kivi_decode_attention")
    return out


def kv_cache_bytes(layers: int, batch: int, seq_len: int, kv_heads: int,
                   head_dim: int, bytes_num: int, bytes_den: int = 1) -> float:
    """2*L*B*T*H_kv*d_h*bytes, bytes = bytes_num/bytes_den."""
    return _load().oracle_kv_cache_bytes(layers, batch, seq_len, kv_heads,
                                         head_dim, bytes_num, bytes_den)


def kv8_scale_bytes(layers: int, batch: int, seq_len: int, kv_heads: int) -> float:
    """Bytes of fp32 scales the INT8 cache adds (one per token, head, K/V)."""
    return _load().oracle_kv8_scale_bytes(layers, batch, seq_len, kv_heads)
