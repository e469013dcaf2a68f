"""GPU edge cases and properties of the decode path (through the C ABI).

  * ragged and degenerate contexts (0, 1, 15, 16, 17, chunk-1, chunk,
    chunk+1, several chunks), every group size (1, 2, 4, 8), no-split and
    split launches with several chunk sizes, against the oracle;
  * physical block permutation gives a bit-identical output;
  * sequences sharing prefix blocks with equal suffixes give bit-identical
    outputs, equal to a private copy of the same tokens;
  * split and no-split launches agree within 1e-5 (fp32 output);
  * kv8_split_reduce called on its own reproduces the fused call;
  * poisoned (NaN-scale, code-127) unused slots never reach the output.
"""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("needs a GPU", allow_module_level=True)

from tests import gpu_util as U  # noqa: E402

RAGGED = [0, 1, 15, 16, 17, 255, 511, 512, 513, 1000, 1537]


@pytest.fixture(scope="module")
def pk():
    from paged_int8_kv_b200 import build
    build.build()
    import paged_int8_kv_b200 as m
    yield m
    assert m.kv8_read_device_status(clear=True) == 0


def _ref(oracle_mod, w):
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    return oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                       w.context_lens)


@pytest.mark.parametrize("kind", [1, 2, 3, 4],
                         ids=["cudacore", "mmasync", "tcgen05", "mma_i8"])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 4), (8, 2), (16, 2), (4, 1)])
@pytest.mark.parametrize("chunk", [0, 16, 512])
def test_ragged_groups_chunks(pk, oracle_mod, hq, hkv, chunk, kind):
    w = W.make_workload("ragged", 2000 + hq * 10 + hkv, RAGGED, hq, hkv,
                        extra_blocks=7, outliers=(3, 10.0), chunk_tokens=chunk)
    ref = _ref(oracle_mod, w)
    cache, q, bt, cl = U.device_inputs(w)
    for dt, bf in ((torch.float32, False), (torch.bfloat16, True)):
        gpu = U.gpu_decode(cache, q, bt, cl, w, chunk_tokens=chunk,
                           out_dtype=dt, form=kind)
        U.assert_close(gpu, ref, bf16=bf)
        if not bf:
            assert np.abs(gpu - ref).max() < 1e-4
        assert np.all(gpu[0] == 0.0)  # empty context -> zeros


@pytest.mark.parametrize("scale", [2.0 ** -40, 1.0, 2.0 ** 20])
def test_tensorcore_extreme_magnitudes(pk, oracle_mod, scale):
    # q and V far from unit scale exercise the power-of-two normalisation of
    # q and of the fp16 probabilities in the tensor-core form
    w = W.make_workload("mag", 2100, [700, 64, 1], 16, 4, extra_blocks=2)
    q = W.bf16_bits_to_f32(w.q()) * np.float32(scale)
    w._q = W.f32_to_bf16_bits(q)
    base = w.private_kv

    def scaled(b, _base=base):
        k, v = _base(b)
        vf = W.bf16_bits_to_f32(v) * np.float32(1.0 / scale if scale > 1 else scale)
        return k, W.f32_to_bf16_bits(vf)
    w.private_kv = scaled
    ref = _ref(oracle_mod, w)
    cache, qd, bt, cl = U.device_inputs(w)
    for kind in (1, 2, 3, 4):
        gpu = U.gpu_decode(cache, qd, bt, cl, w, chunk_tokens=256, form=kind)
        denom = max(np.abs(ref).max(), 1e-30)
        assert np.abs(gpu - ref).max() / denom < 1e-4, kind


def test_tensorcore_matches_cudacore(pk):
    w = W.make_workload("kinds", 2200, [5000, 3000, 17], 64, 8, extra_blocks=1,
                        outliers=(4, 8.0))
    cache, q, bt, cl = U.device_inputs(w)
    outs = []
    for kind in (1, 2, 3, 4):
        outs.append(U.gpu_decode(cache, q, bt, cl, w, chunk_tokens=512,
                                 form=kind))
    for o in outs[1:]:
        assert np.abs(outs[0] - o).max() < 1e-4


def test_block_permutation_bit_identical(pk):
    lens = [300, 77, 1024]
    a = W.make_workload("perm", 3001, lens, 16, 4, extra_blocks=5)
    b = W.make_workload("perm", 3001, lens, 16, 4, extra_blocks=5)
    # same tokens, different physical placement
    rng = np.random.default_rng(5)
    perm = rng.permutation(b.num_blocks).astype(np.int32)
    b.block_tables = perm[a.block_tables]
    outs = []
    for w in (a, b):
        cache, q, bt, cl = U.device_inputs(w)
        outs.append(U.gpu_decode(cache, q, bt, cl, w, chunk_tokens=256))
    assert np.array_equal(outs[0], outs[1])


def test_prefix_sharing_bit_identical(pk, oracle_mod):
    # sequences 0..2 share a 64-token prefix; 1 and 2 have the same suffix
    # length and seed-independent identical data is arranged below
    w = W.make_workload("pre", 3002, [64 + 40, 64 + 40, 64 + 40, 64 + 40], 8, 2,
                        prefix_group=[0, 0, 0, -1], prefix_len=64,
                        chunk_tokens=32)
    # make suffix data of sequences 1, 2 and the private copy in 3 equal to 0's
    base_k, base_v = w.private_kv(0)
    pre_k, pre_v = w.prefix_kv(0)
    w.private_kv = lambda b, _k=base_k, _v=base_v, _pk=pre_k, _pv=pre_v: (
        (np.concatenate([_pk, _k]), np.concatenate([_pv, _v])) if b == 3
        else (_k, _v))
    qb = w.q()
    qb[:] = qb[0:1]
    cache, q, bt, cl = U.device_inputs(w)
    out = U.gpu_decode(cache, q, bt, cl, w)
    assert np.array_equal(out[0], out[1]) and np.array_equal(out[0], out[2])
    assert np.array_equal(out[0], out[3])
    ref = _ref(oracle_mod, w)
    U.assert_close(out, ref, bf16=False)


def test_split_vs_nosplit_and_standalone_reduce(pk):
    w = W.make_workload("split", 3003, [4096, 2500, 700, 33], 32, 8,
                        extra_blocks=3)
    cache, q, bt, cl = U.device_inputs(w)
    one = U.gpu_decode(cache, q, bt, cl, w, chunk_tokens=0)
    for ct in (16, 256, 512, 2048):
        s = U.gpu_decode(cache, q, bt, cl, w, chunk_tokens=ct)
        assert np.abs(s - one).max() <= 1e-5, ct
    # the standalone reduce over the same workspace gives the same rows
    out = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    ws = cache.workspace(w.batch, w.num_q_heads, w.max_context_len, 512)
    pk.kv8_paged_decode_attention(q, cache.k_cache, cache.v_cache,
                                  cache.k_scales, cache.v_scales, bt, cl, out,
                                  w.max_context_len, chunk_tokens=512,
                                  workspace=ws)
    fused = out.clone()
    out2 = fused.clone()
    long_rows = [b for b in range(w.batch) if int(w.context_lens[b]) > 512]
    out2[long_rows] = 0.0
    pk.kv8_split_reduce(ws, cl, out2, w.max_context_len, 512)
    torch.cuda.synchronize()
    assert torch.equal(out2, fused)


def test_error_codes_on_gpu(pk):
    import paged_int8_kv_b200 as m
    w = W.make_workload("err", 3004, [600], 8, 2)
    cache, q, bt, cl = U.device_inputs(w)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.Kv8Error) as e:
        m.kv8_paged_decode_attention(q, cache.k_cache, cache.v_cache,
                                     cache.k_scales, cache.v_scales, bt, cl,
                                     out, w.max_context_len, chunk_tokens=256,
                                     workspace=small)
    assert e.value.status == m.KV8_ERR_WORKSPACE
