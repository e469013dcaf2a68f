"""kv8_paged_decode_attention_append (one launch: quantise the step's new
tokens into the cache, then decode) against the two-call path and the oracle:

  * the cache it leaves (codes and scales) equals, bit for bit, the cache
    kv8_quantize_append leaves for the same tokens;
  * its output equals kv8_paged_decode_attention's on that cache bit for bit
    (same kernel arithmetic, same split), and the oracle within the decode
    tolerance;
  * split and unsplit launches, ragged and empty contexts, groups 1 to 8.
"""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("needs a GPU", allow_module_level=True)

from tests import gpu_util as U  # noqa: E402


@pytest.fixture(scope="module")
def pk():
    from paged_int8_kv_b200 import build
    build.build()
    import paged_int8_kv_b200 as m
    yield m
    assert m.kv8_read_device_status(clear=True) == 0


def _ragged(hq, hkv):
    return W.make_workload(f"app_g{hq // hkv}", 5100 + hq + hkv,
                           [1, 15, 16, 17, 0, 300, 1000, 33], hq, hkv,
                           extra_blocks=5, outliers=(3, 10.0))


CASES = {
    "tiny": W.tiny,
    "llama8b_b32": W.llama8b_b32,
    "ragged_g1": lambda: _ragged(8, 8),
    "ragged_g4": lambda: _ragged(16, 4),
    "ragged_g8": lambda: _ragged(16, 2),
}


def _cache_without_step(w):
    from paged_int8_kv_b200 import PagedKV8Cache
    from paged_int8_kv_b200.runtime import fill_from_host
    cache = PagedKV8Cache(w.num_blocks, w.num_kv_heads, device="cuda")
    fill_from_host(cache, w.fill_segments())
    return cache


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("chunk", [0, 64, 512])
def test_append_matches_two_calls_and_oracle(pk, oracle_mod, name, chunk):
    w = CASES[name]()
    kn, vn, sl = w.step_tokens()
    k_new = torch.from_numpy(kn).view(torch.bfloat16).cuda()
    v_new = torch.from_numpy(vn).view(torch.bfloat16).cuda()
    q = torch.from_numpy(w.q()).view(torch.bfloat16).cuda()
    bt = torch.from_numpy(w.block_tables).cuda()
    cl = torch.from_numpy(w.context_lens).cuda()
    mcl = max(w.max_context_len, 1)

    # the two-call path
    a = _cache_without_step(w)
    a.append(k_new, v_new, torch.from_numpy(sl).cuda())
    out_a = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    ws_a = a.workspace(w.batch, w.num_q_heads, mcl, chunk)
    pk.kv8_paged_decode_attention(q, a.k_cache, a.v_cache, a.k_scales, a.v_scales,
                                  bt, cl, out_a, mcl, chunk_tokens=chunk,
                                  workspace=ws_a)
    # the fused call
    b = _cache_without_step(w)
    out_b = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    ws_b = b.workspace(w.batch, w.num_q_heads, mcl, chunk)
    pk.kv8_paged_decode_attention_append(q, k_new, v_new, b.k_cache, b.v_cache,
                                         b.k_scales, b.v_scales, bt, cl, out_b,
                                         mcl, chunk_tokens=chunk, workspace=ws_b)
    torch.cuda.synchronize()
    assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.v_cache, b.v_cache)
    assert torch.equal(a.k_scales.view(torch.int32), b.k_scales.view(torch.int32))
    assert torch.equal(a.v_scales.view(torch.int32), b.v_scales.view(torch.int32))
    assert torch.equal(out_a, out_b)
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    ref = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    U.assert_close(out_b.cpu().numpy(), ref, bf16=False)


def test_runtime_step_is_the_fused_call(pk, oracle_mod):
    # PagedKV8Cache.step wraps kv8_paged_decode_attention_append
    w = W.tiny()
    kn, vn, _ = w.step_tokens()
    c = _cache_without_step(w)
    q = torch.from_numpy(w.q()).view(torch.bfloat16).cuda()
    out = c.step(q, torch.from_numpy(kn).view(torch.bfloat16).cuda(),
                 torch.from_numpy(vn).view(torch.bfloat16).cuda(),
                 torch.from_numpy(w.block_tables).cuda(),
                 torch.from_numpy(w.context_lens).cuda(), w.max_context_len,
                 chunk_tokens=64, out_dtype=torch.float32)
    torch.cuda.synchronize()
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    assert np.array_equal(c.k_cache.cpu().numpy(), kc)
    ref = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    U.assert_close(out.cpu().numpy(), ref, bf16=False)
