"""kv8_paged_decode_attention_noalloc, called through the C ABI.

Some callers cannot allocate device memory: code running inside a host
framework that owns the whole GPU memory budget (a serving engine that
reserves nearly all of it for its KV pool up front), a plugin or custom op
whose host offers no workspace hook, or a latency-critical path that must not
call cudaMalloc because it can synchronise the device.  For them the split-K
decode keeps its chunk partials in the library's fixed per-device scratch
array instead of a caller workspace.

The test checks, on two calls in a row, that the entry point returns exactly
what the allocating entry point returns on the same inputs (the same kernel
with the same split and merge order, so bit for bit), that both agree with
the CPU oracle within the parity tolerance, and that a split needing more
scratch than the fixed array holds is refused before anything runs.

The file name sorts last so that a run stopping at the first failure has
run every other test first; it needs nothing from the other test files.
"""
import ctypes

import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("needs a GPU", allow_module_level=True)

from tests import gpu_util as U  # noqa: E402

NOALLOC_LIMIT = 16 << 20  # KV8_NOALLOC_WORKSPACE_BYTES in include/kv8.h

_P, _I32, _I64, _F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float


def _lib():
    from paged_int8_kv_b200 import build
    build.build()
    lib = ctypes.CDLL(build.LIB)
    lib.kv8_paged_decode_attention_noalloc.restype = _I32
    lib.kv8_paged_decode_attention_noalloc.argtypes = [
        _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I64,
        _I32, _F32, _I32, _P, _I32, _P]
    lib.kv8_paged_decode_attention.restype = _I32
    lib.kv8_paged_decode_attention.argtypes = [
        _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I64,
        _I32, _F32, _I32, _P, ctypes.c_size_t, _P, _I32, _P]
    lib.kv8_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.kv8_decode_workspace_bytes.argtypes = [_I32, _I32, _I32, _I32, _I32]
    lib.kv8_read_device_status.restype = _I32
    lib.kv8_read_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), _I32]
    return lib


def _common(q, cache, bt, cl, maxlen, chunk):
    B, hq, d = q.shape
    nb, hkv, bs, _ = cache.k_cache.shape
    return (q.data_ptr(), cache.k_cache.data_ptr(), cache.v_cache.data_ptr(),
            cache.k_scales.data_ptr(), cache.v_scales.data_ptr(),
            bt.data_ptr(), cl.data_ptr(), B, hq, hkv, d, bs, bt.shape[1], nb,
            maxlen, 0.0, chunk)


def _odt(out):
    return 1 if out.dtype == torch.float32 else 0


def _status(lib):
    v = ctypes.c_uint32(0)
    assert lib.kv8_read_device_status(ctypes.byref(v), 1) == 0
    return v.value


def test_noalloc_matches_allocating_entry_point(oracle_mod):
    lib = _lib()
    w = W.make_workload("noalloc", 4242, [4096, 2500, 700, 33, 1537, 0], 32, 8,
                        extra_blocks=3, outliers=(3, 10.0))
    chunk = 256
    need = lib.kv8_decode_workspace_bytes(w.batch, w.num_q_heads, 128,
                                          w.max_context_len, chunk)
    assert 0 < need <= NOALLOC_LIMIT
    cache, q, bt, cl = U.device_inputs(w)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    args = _common(q, cache, bt, cl, w.max_context_len, chunk)
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    exact = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                        w.context_lens)
    for dt in (torch.float32, torch.bfloat16):
        ref = torch.full(q.shape, float("nan"), dtype=dt, device="cuda")
        rc = lib.kv8_paged_decode_attention(*args, ws.data_ptr(), need,
                                            ref.data_ptr(), _odt(ref), stream)
        assert rc == 0
        for _ in range(2):  # two calls in a row share the scratch array
            out = torch.full(q.shape, float("nan"), dtype=dt, device="cuda")
            rc = lib.kv8_paged_decode_attention_noalloc(
                *args, out.data_ptr(), _odt(out), stream)
            assert rc == 0
            torch.cuda.synchronize()
            # same kernel, same split, same merge order: bit for bit
            assert torch.equal(out.view(torch.int16 if dt == torch.bfloat16
                                        else torch.int32),
                               ref.view(torch.int16 if dt == torch.bfloat16
                                        else torch.int32))
            got = out.float().cpu().numpy()
            U.assert_close(got, exact, bf16=(dt == torch.bfloat16))
    assert _status(lib) == 0


def test_noalloc_rejects_split_beyond_limit():
    lib = _lib()
    # batch 64 x 32 heads x 64 chunks of partials (68 MB) > 16 MiB: refused on
    # the host before any launch.  The stand-in inputs are harmless even if a
    # launch did happen: every table entry is block 0 of the 16-block cache
    # and every device-side context length is 0 (no page read, no partial).
    B, hq, hkv, maxlen, chunk = 64, 32, 8, 32768, 512
    need = lib.kv8_decode_workspace_bytes(B, hq, 128, maxlen, chunk)
    assert need > NOALLOC_LIMIT
    from paged_int8_kv_b200 import PagedKV8Cache
    cache = PagedKV8Cache(16, hkv, poison=False)
    q = torch.zeros((B, hq, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((B, maxlen // 16), dtype=torch.int32, device="cuda")
    cl = torch.zeros((B,), dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    rc = lib.kv8_paged_decode_attention_noalloc(
        *_common(q, cache, bt, cl, maxlen, chunk), out.data_ptr(), 0,
        torch.cuda.current_stream().cuda_stream)
    assert rc == 3  # KV8_ERR_WORKSPACE
    torch.cuda.synchronize()
    # a larger chunk needs fewer partials and fits
    assert lib.kv8_decode_workspace_bytes(B, hq, 128, maxlen, 4096) <= NOALLOC_LIMIT
