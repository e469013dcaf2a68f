"""kv8_paged_extend_attention (prefill / chunked-prefill attention over the
paged INT8 cache, on the tcgen05 tensor cores) against the oracle's causal
extend attention, through the C ABI.

  * mixed batches: a whole prompt (every cached token is new), a one-row
    extension (the decode case), a long extension of a longer cache, ragged
    lengths that end inside a page and inside a key tile; every GQA group
    size; fp32 and bf16 output, |gpu - oracle| <= 2e-3 (+ half a bf16 ulp);
  * one new row per sequence agrees with the decode entry point;
  * a 4096-token cache extended by 1000 rows (many key and query tiles);
  * the extend bench's own workload at full size, sampled rows.
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


def _extend(pk, w, new, seed, out_dtype=torch.float32):
    cache, _, bt, cl = U.device_inputs(w)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    rng = np.random.default_rng([seed, 9])
    qh = W.f32_to_bf16_bits(rng.standard_normal(
        (int(qs[-1]), w.num_q_heads, 128), dtype=np.float32))
    q = torch.from_numpy(qh).view(torch.bfloat16).cuda()
    out = torch.full(q.shape, float("nan"), dtype=out_dtype, device="cuda")
    pk.kv8_paged_extend_attention(
        q, cache.k_cache, cache.v_cache, cache.k_scales, cache.v_scales, bt,
        cl, torch.from_numpy(qs).cuda(), out, int(max(new)))
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), qh, qs, (cache, bt, cl)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 4), (32, 8), (16, 2)])
def test_extend_mixed_batch(pk, oracle_mod, hq, hkv):
    lens = [40, 300, 1000, 17, 129]
    new = [40, 1, 300, 17, 100]
    w = W.make_workload("ext", 7000 + hq + hkv, lens, hq, hkv, extra_blocks=4,
                        outliers=(3, 10.0))
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    for dt, bf in ((torch.float32, False), (torch.bfloat16, True)):
        got, qh, qs, _ = _extend(pk, w, new, 11, dt)
        ref = oracle_mod.extend_attention(qh, kc, vc, ks, vs, w.block_tables,
                                          w.context_lens, qs)
        err = U.assert_close(got, ref, bf16=bf)
        print(f"extend G={hq // hkv} {dt}: max err {err:.3e}")


def test_extend_one_row_matches_decode(pk, oracle_mod):
    lens = [700, 33, 4000]
    w = W.make_workload("ext1", 7100, lens, 32, 8, extra_blocks=2)
    got, qh, qs, (cache, bt, cl) = _extend(pk, w, [1, 1, 1], 12)
    w._q = qh.reshape(3, 32, 128)
    q = torch.from_numpy(w._q).view(torch.bfloat16).cuda()
    dec = U.gpu_decode(cache, q, bt, cl, w, chunk_tokens=0)
    assert np.abs(got - dec).max() <= 2e-3
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    ref = oracle_mod.decode_attention(w._q, kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    U.assert_close(got, ref, bf16=False)


def test_extend_long(pk, oracle_mod):
    w = W.make_workload("extlong", 7200, [4096], 32, 8, extra_blocks=1)
    got, qh, qs, _ = _extend(pk, w, [1000], 13)
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    # every 37th row (all heads): the oracle one row at a time
    rows = list(range(0, 1000, 37)) + [999]
    for i in rows:
        sub = oracle_mod.extend_attention(
            qh[i:i + 1], kc, vc, ks, vs, w.block_tables,
            np.array([4096 - 1000 + i + 1], dtype=np.int32), np.array([0, 1]))
        U.assert_close(got[i:i + 1], sub, bf16=False)


def test_extend_bench_size_sampled_rows(pk, oracle_mod):
    """The extend bench's workload at full size (batch 4, 32768 cached
    tokens each, the last 2048 new; q drawn as the bench draws it): sampled
    rows of two sequences, all heads, against the oracle one row at a time
    (row i of sequence b sees the first 32768 - 2048 + i + 1 tokens)."""
    T, NEW = 32768, 2048
    w = W.make_workload("llama8b_extend_b4_ctx32k_new2k", 1006, [T] * 4, 32, 8)
    got, qh, qs, _ = _extend(pk, w, [NEW] * 4, 1006)
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    for b in (0, 3):
        for i in (0, 1023, NEW - 1):
            r = int(qs[b]) + i
            sub = oracle_mod.extend_attention(
                qh[r:r + 1], kc, vc, ks, vs, w.block_tables[b:b + 1],
                np.array([T - NEW + i + 1], dtype=np.int32), np.array([0, 1]))
            U.assert_close(got[r:r + 1], sub, bf16=False)
    assert np.all(np.isfinite(got))
