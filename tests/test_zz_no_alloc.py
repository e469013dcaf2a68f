"""kv8_paged_decode_attention_noalloc, called through the C ABI.

This entry point serves callers that cannot allocate device memory (a host
framework that owns the whole GPU memory budget, a plugin without a
workspace hook, code that must not risk cudaMalloc's device
synchronisation): it keeps the split-K partials in the library's fixed
per-device scratch array instead of a caller workspace.  The test checks, on
two calls in a row, that it returns what the allocating entry point returns
on the same inputs, and that a split needing more scratch than the fixed
array holds is refused before anything runs.

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


def _c_noalloc(lib, q, cache, bt, cl, out, maxlen, chunk):
    f = lib.kv8_paged_decode_attention_noalloc
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f.restype = i32
    f.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i64, i32,
                  ctypes.c_float, i32, P, i32, P]
    B, hq, d = q.shape
    nb, hkv, bs, _ = cache.k_cache.shape
    return f(q.data_ptr(), cache.k_cache.data_ptr(), cache.v_cache.data_ptr(),
             cache.k_scales.data_ptr(), cache.v_scales.data_ptr(),
             bt.data_ptr(), cl.data_ptr(), B, hq, hkv, d, bs, bt.shape[1], nb,
             maxlen, 0.0, chunk, out.data_ptr(),
             1 if out.dtype == torch.float32 else 0,
             torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_allocating_entry_point():
    from paged_int8_kv_b200 import build
    build.build()
    import paged_int8_kv_b200 as pk
    lib = ctypes.CDLL(pk.LIB_PATH)
    w = W.make_workload("noalloc", 4242, [4096, 2500, 700, 33, 1537, 0], 32, 8,
                        extra_blocks=3, outliers=(3, 10.0))
    chunk = 256
    need = pk.kv8_decode_workspace_bytes(w.batch, w.num_q_heads, 128,
                                         w.max_context_len, chunk)
    assert 0 < need <= NOALLOC_LIMIT
    cache, q, bt, cl = U.device_inputs(w)
    for dt in (torch.float32, torch.bfloat16):
        ref = cache.decode(q, bt, cl, w.max_context_len, chunk_tokens=chunk,
                           out_dtype=dt)
        torch.cuda.synchronize()
        ref = ref.float().cpu().numpy()
        for _ in range(2):  # two calls in a row share the scratch array
            out = torch.full(q.shape, float("nan"), dtype=dt, device="cuda")
            rc = _c_noalloc(lib, q, cache, bt, cl, out, w.max_context_len, chunk)
            assert rc == 0, pk.kv8_status_string(rc)
            torch.cuda.synchronize()
            got = out.float().cpu().numpy()
            assert np.all(np.isfinite(got))
            err = np.abs(got.astype(np.float64) - ref)
            assert err.max() <= 2e-3  # the tolerance the parity tests use
    assert pk.kv8_read_device_status(clear=True) == 0


def test_noalloc_rejects_split_beyond_limit():
    from paged_int8_kv_b200 import build
    build.build()
    import paged_int8_kv_b200 as pk
    lib = ctypes.CDLL(pk.LIB_PATH)
    # batch 64 x 32 heads x 64 chunks of partials (68 MB) > 16 MiB: refused on
    # the host before any launch, so the tiny stand-in buffers are never read
    w = W.make_workload("big", 1, [32768] * 64, 32, 8, num_blocks=64 * 2048)
    need = pk.kv8_decode_workspace_bytes(64, 32, 128, 32768, 512)
    assert need > NOALLOC_LIMIT
    cache = pk.PagedKV8Cache(16, 8, poison=False)
    q = torch.zeros((64, 32, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.from_numpy(w.block_tables).cuda()
    cl = torch.from_numpy(w.context_lens).cuda()
    out = torch.empty_like(q)
    rc = _c_noalloc(lib, q, cache, bt, cl, out, 32768, 512)
    assert rc == pk.KV8_ERR_WORKSPACE
    # a larger chunk needs fewer partials and fits
    assert pk.kv8_decode_workspace_bytes(64, 32, 128, 32768, 4096) <= NOALLOC_LIMIT
