"""The decode kernel's bounded waits give up cleanly (no fault, no hang).

Uses the test-hook build of the library (libkv8_testhooks.so, the same
sources compiled with -DKV8_TEST_HOOKS): there a wait for a page gives up
after a few milliseconds, and a switch makes warp 0 of CTA 0 arm its first
page's mbarrier without issuing that page's copies.  Nothing is copied
wrongly and nothing faults: the wait simply never completes.  The launch
must still return KV8_OK, finish, and leave bit 0 (wait given up) in the
device status word; with the switch off, the next call on the same context
returns the oracle's result with a clean status.
"""
import ctypes

import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("needs a GPU", allow_module_level=True)

from tests import gpu_util as U  # noqa: E402

_P, _I32, _I64, _F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float


@pytest.fixture(scope="module")
def hooks():
    from paged_int8_kv_b200 import build
    lib = ctypes.CDLL(build.build(test_hooks=True))
    lib.kv8_paged_decode_attention_form.restype = _I32
    lib.kv8_paged_decode_attention_form.argtypes = [
        _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I64,
        _I32, _F32, _I32, _P, ctypes.c_size_t, _P, _I32, _I32, _P]
    lib.kv8_read_device_status.restype = _I32
    lib.kv8_read_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), _I32]
    lib.kv8_test_skip_first_copy.restype = _I32
    lib.kv8_test_skip_first_copy.argtypes = [_I32]
    yield lib
    lib.kv8_test_skip_first_copy(0)


def _status(lib):
    v = ctypes.c_uint32(0)
    assert lib.kv8_read_device_status(ctypes.byref(v), 1) == 0
    return v.value


def _decode(lib, cache, q, bt, cl, w, out, ws, form):
    B, hq, d = q.shape
    nb, hkv, bs, _ = cache.k_cache.shape
    return lib.kv8_paged_decode_attention_form(
        q.data_ptr(), cache.k_cache.data_ptr(), cache.v_cache.data_ptr(),
        cache.k_scales.data_ptr(), cache.v_scales.data_ptr(), bt.data_ptr(),
        cl.data_ptr(), B, hq, hkv, d, bs, bt.shape[1], nb, w.max_context_len,
        0.0, 256, ws.data_ptr(), ws.numel(), out.data_ptr(), 1, form,
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("form", [1, 2, 4], ids=["cudacore", "mmasync", "mma_i8"])
def test_wait_gives_up_then_clean_call(hooks, oracle_mod, form):
    w = W.make_workload("giveup", 5151, [1000, 300, 77, 0], 16, 4,
                        extra_blocks=2)
    cache, q, bt, cl = U.device_inputs(w)
    ws = cache.workspace(w.batch, w.num_q_heads, w.max_context_len, 256)
    out = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    _status(hooks)  # start clean
    assert hooks.kv8_test_skip_first_copy(1) == 0
    assert _decode(hooks, cache, q, bt, cl, w, out, ws, form) == 0
    torch.cuda.synchronize()  # the launch ends: the stalled warp gave up
    assert _status(hooks) & 1 == 1
    assert hooks.kv8_test_skip_first_copy(0) == 0
    # the context is healthy and the next call is exact again
    out.zero_()
    assert _decode(hooks, cache, q, bt, cl, w, out, ws, form) == 0
    torch.cuda.synchronize()
    assert _status(hooks) == 0
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    ref = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    U.assert_close(out.cpu().numpy(), ref, bf16=False)
