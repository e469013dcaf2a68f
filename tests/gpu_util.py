"""Helpers shared by the GPU tests: fill a device cache from a workload, run
the CUDA path, and build the oracle's view of the same inputs."""
from __future__ import annotations

import math

import numpy as np
import torch

import workloads as W


def device_inputs(w: W.Workload, device="cuda"):
    from paged_int8_kv_b200 import PagedKV8Cache
    from paged_int8_kv_b200.runtime import fill_from_host
    cache = PagedKV8Cache(w.num_blocks, w.num_kv_heads, device=device)
    fill_from_host(cache, w.fill_segments())
    k, v, s = w.step_tokens()
    fill_from_host(cache, [(k, v, s)])
    bt = torch.from_numpy(w.block_tables).to(device)
    cl = torch.from_numpy(w.context_lens).to(device)
    q = torch.from_numpy(w.q()).view(torch.bfloat16).to(device)
    return cache, q, bt, cl


def gpu_decode(cache, q, bt, cl, w: W.Workload, chunk_tokens=None,
               out_dtype=torch.float32, form=0):
    ct = w.chunk_tokens if chunk_tokens is None else chunk_tokens
    out = cache.decode(q, bt, cl, w.max_context_len, chunk_tokens=ct,
                       out_dtype=out_dtype, form=form)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


def oracle_full_cache(oracle, w: W.Workload):
    """The oracle's own paged cache for every token of the workload."""
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    kc = np.full(shape, 127, dtype=np.int8)
    vc = np.full(shape, 127, dtype=np.int8)
    ks = np.full(shape[:3], np.nan, dtype=np.float32)
    vs = np.full(shape[:3], np.nan, dtype=np.float32)
    segs = list(w.fill_segments()) + [w.step_tokens()]
    for k, v, s in segs:
        oracle.quantize_append(k, s, kc, ks)
        oracle.quantize_append(v, s, vc, vs)
    return kc, vc, ks, vs


def oracle_sequence_cache(oracle, w: W.Workload, b: int):
    """A private, contiguously numbered cache holding sequence b only."""
    k, v = w.sequence_kv(b)
    n = k.shape[0]
    nblk = max(1, math.ceil(n / w.block_size))
    shape = (nblk, w.num_kv_heads, w.block_size, w.head_dim)
    kc = np.full(shape, 127, dtype=np.int8)
    vc = np.full(shape, 127, dtype=np.int8)
    ks = np.full(shape[:3], np.nan, dtype=np.float32)
    vs = np.full(shape[:3], np.nan, dtype=np.float32)
    slots = np.arange(n, dtype=np.int64)
    oracle.quantize_append(k, slots, kc, ks)
    oracle.quantize_append(v, slots, vc, vs)
    table = np.arange(nblk, dtype=np.int32)[None, :]
    return kc, vc, ks, vs, table


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp at |x| (for the bf16-output comparison)."""
    a = np.abs(x).astype(np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 8)


def assert_close(gpu: np.ndarray, ref: np.ndarray, bf16: bool, tol=2e-3):
    err = np.abs(gpu.astype(np.float64) - ref)
    bound = tol + (bf16_half_ulp(ref) if bf16 else 0.0)
    bad = err > bound
    assert not bad.any(), (
        f"{int(bad.sum())} elements outside tolerance; max err {err.max():.3e}")
    return float(err.max())


def oracle_kivi_sequence(oracle, w: W.Workload, b: int):
    """The oracle's private KIVI cache for sequence b (contiguously numbered
    blocks), built as the fill and step calls build a device cache: every
    token but the last, then the last.  Returns (cache, table)."""
    k, v = w.sequence_kv(b)
    n = k.shape[0]
    nblk = max(1, math.ceil(n / w.block_size))
    table = np.arange(nblk, dtype=np.int32)[None, :]
    c = oracle.KiviCache(nblk, w.num_kv_heads, 1)
    if n > 1:
        oracle.kivi_append(c, k[:-1], v[:-1], np.array([0, n - 1]),
                           np.array([n - 1]), table)
    if n > 0:
        oracle.kivi_append(c, k[-1:], v[-1:], np.array([0, 1]), np.array([n]),
                           table)
    return c, table


def oracle_int4_sequence(oracle, w: W.Workload, b: int):
    """The oracle's private INT4 cache for sequence b (contiguously numbered
    blocks): (k codes, v codes, k scales, v scales, table)."""
    k, v = w.sequence_kv(b)
    n = k.shape[0]
    nblk = max(1, math.ceil(n / w.block_size))
    shape = (nblk, w.num_kv_heads, w.block_size, w.head_dim // 2)
    kc = np.zeros(shape, dtype=np.uint8)
    vc = np.zeros(shape, dtype=np.uint8)
    ks = np.zeros(shape[:3], dtype=np.float32)
    vs = np.zeros(shape[:3], dtype=np.float32)
    slots = np.arange(n, dtype=np.int64)
    oracle.quantize_append_int4(k, slots, kc, ks)
    oracle.quantize_append_int4(v, slots, vc, vs)
    return kc, vc, ks, vs, np.arange(nblk, dtype=np.int32)[None, :]
