"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

  * quantise-append: codes and scales bit-exact, on every slot of the tiny,
    batch-32, pruned and prefix-shared workloads and on sampled sequences of
    the batch-64 x 32K workload;
  * decode attention: every (sequence, query head) of the small workloads and
    sampled ones of the 32K workload, in the split-K launch the bench times,
    within the tolerance stated by the method's target: |gpu - oracle| <= 2e-3
    for fp32 output, plus half a bf16 ulp of the exact value for bf16 output
    (the rounding of the output itself); both for the default decode form
    and for the tcgen05 form.
"""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("needs a GPU", allow_module_level=True)

from tests import gpu_util as U  # noqa: E402

SMALL = ["tiny", "llama8b_b32", "pruned_compact", "prefix_shared_70b"]


def _u32(a):
    return np.ascontiguousarray(a).view(np.uint32)


@pytest.fixture(scope="module")
def built():
    from paged_int8_kv_b200 import build
    build.build()
    import paged_int8_kv_b200 as pk
    yield pk
    assert pk.kv8_read_device_status(clear=True) == 0


_cache = {}


def _setup(name, oracle_mod):
    if name not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        w = W.NAMED[name]()
        dev = U.device_inputs(w)
        _cache[name] = (w, dev, U.oracle_full_cache(oracle_mod, w))
    return _cache[name]


@pytest.mark.parametrize("name", SMALL)
def test_quantize_bit_exact(built, oracle_mod, name):
    w, (cache, q, bt, cl), (kc, vc, ks, vs) = _setup(name, oracle_mod)
    assert np.array_equal(cache.k_cache.cpu().numpy(), kc)
    assert np.array_equal(cache.v_cache.cpu().numpy(), vc)
    assert np.array_equal(_u32(cache.k_scales.cpu().numpy()), _u32(ks))
    assert np.array_equal(_u32(cache.v_scales.cpu().numpy()), _u32(vs))


KINDS = pytest.mark.parametrize("kind", [0, 2, 3, 4],
                                ids=["default", "mma_f16pv", "tcgen05", "mma_i8"])


@KINDS
@pytest.mark.parametrize("name", SMALL)
@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_decode_all_pairs(built, oracle_mod, name, out_dtype, kind):
    w, (cache, q, bt, cl), (kc, vc, ks, vs) = _setup(name, oracle_mod)
    ref = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    dt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    gpu = U.gpu_decode(cache, q, bt, cl, w, out_dtype=dt, form=kind)
    U.assert_close(gpu, ref, bf16=(out_dtype == "bf16"))
    if out_dtype == "f32":
        # the fp32 path is far inside the tolerance: a regression shows here
        assert np.abs(gpu - ref).max() < 1e-4


@pytest.fixture(scope="module")
def big(built, oracle_mod):
    _cache.clear()
    torch.cuda.empty_cache()
    w = W.llama8b_b64_32k()
    dev = U.device_inputs(w)
    yield w, dev
    del dev
    torch.cuda.empty_cache()


BIG_SEQS = [0, 37, 63]


def test_big_quantize_sampled_sequences(big, oracle_mod):
    w, (cache, q, bt, cl) = big
    for b in BIG_SEQS:
        kc, vc, ks, vs, _ = U.oracle_sequence_cache(oracle_mod, w, b)
        blocks = torch.from_numpy(w.block_tables[b].astype(np.int64)).cuda()
        assert np.array_equal(cache.k_cache[blocks].cpu().numpy(), kc)
        assert np.array_equal(cache.v_cache[blocks].cpu().numpy(), vc)
        assert np.array_equal(_u32(cache.k_scales[blocks].cpu().numpy()), _u32(ks))
        assert np.array_equal(_u32(cache.v_scales[blocks].cpu().numpy()), _u32(vs))


@KINDS
@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_big_decode_sampled(big, oracle_mod, out_dtype, kind):
    w, (cache, q, bt, cl) = big
    dt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    gpu = U.gpu_decode(cache, q, bt, cl, w, out_dtype=dt, form=kind)
    rng = np.random.default_rng(77)
    for b in BIG_SEQS:
        kc, vc, ks, vs, table = U.oracle_sequence_cache(oracle_mod, w, b)
        heads = sorted(rng.choice(w.num_q_heads, 8, replace=False).tolist())
        ref = oracle_mod.decode_attention(
            w.q()[b:b + 1], kc, vc, ks, vs, table, w.context_lens[b:b + 1],
            pairs=[(0, h) for h in heads])
        U.assert_close(gpu[b, heads], ref, bf16=(out_dtype == "bf16"))
    # properties over every row: finite, and no row is the poison pattern
    assert np.all(np.isfinite(gpu))
