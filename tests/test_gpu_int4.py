"""GPU parity of the INT4 cache variant against the CPU oracle.

  * kv8_int4_quantize_append: packed nibbles and scales bit-exact against
    the oracle's INT4 quantise-append on every slot of the workloads;
  * kv8_int4_paged_decode_attention: every (sequence, query head) against
    the oracle's fp64 attention over the dequantised INT4 cache, within the
    decode tolerance (2e-3 for fp32 output, plus half a bf16 ulp for bf16
    output), for groups of 1, 2 and 4 query heads, split and unsplit, with
    ragged and empty contexts;
  * groups of 8 (two sub-groups of 4 heads per KV head): the prefix-shared
    70B batch and ragged contexts.
"""
import itertools

import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU machine
    pytest.skip("needs a GPU", allow_module_level=True)

from tests import gpu_util as U  # noqa: E402

POISON_BYTE = 0xFF  # nibbles 15/15 (code +7) in slots no sequence uses


@pytest.fixture(scope="module")
def built():
    from paged_int8_kv_b200 import build
    build.build()
    import paged_int8_kv_b200 as pk
    yield pk
    assert pk.kv8_read_device_status(clear=True) == 0


def _ragged_g(group):
    return W.make_workload(f"ragged_g{group}", 1100 + group,
                           [1, 15, 16, 17, 0, 300, 1000, 33], 4 * group, 4,
                           extra_blocks=5, outliers=(3, 10.0),
                           description="ragged lengths incl. 0, 1, 15..17")


CASES = {
    "tiny": W.tiny,
    "llama8b_b32": W.llama8b_b32,
    "pruned_compact": W.pruned_compact,
    "ragged_g1": lambda: _ragged_g(1),
    "ragged_g2": lambda: _ragged_g(2),
    "ragged_g4": lambda: _ragged_g(4),
    "ragged_g8": lambda: _ragged_g(8),
    "prefix_shared_70b": W.prefix_shared_70b,
}

_cache = {}


def _segments(w):
    return list(w.fill_segments()) + [w.step_tokens()]


def _device_int4(pk, w, segments=None):
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim // 2)
    kc = torch.full(shape, POISON_BYTE, dtype=torch.uint8, device="cuda")
    vc = torch.full(shape, POISON_BYTE, dtype=torch.uint8, device="cuda")
    ks = torch.full(shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    vs = torch.full(shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    for k, v, s in (_segments(w) if segments is None else segments):
        if s.shape[0] == 0:
            continue
        kt = torch.from_numpy(k).view(torch.bfloat16).cuda()
        vt = torch.from_numpy(v).view(torch.bfloat16).cuda()
        st = torch.from_numpy(s).cuda()
        pk.kv8_int4_quantize_append(kt, vt, st, kc, vc, ks, vs)
    torch.cuda.synchronize()
    return kc, vc, ks, vs


def _oracle_int4(oracle, w):
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim // 2)
    kc = np.full(shape, POISON_BYTE, dtype=np.uint8)
    vc = np.full(shape, POISON_BYTE, dtype=np.uint8)
    ks = np.full(shape[:3], np.nan, dtype=np.float32)
    vs = np.full(shape[:3], np.nan, dtype=np.float32)
    for k, v, s in _segments(w):
        oracle.quantize_append_int4(k, s, kc, ks)
        oracle.quantize_append_int4(v, s, vc, vs)
    return kc, vc, ks, vs


def _setup(pk, oracle, name):
    if name not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        w = CASES[name]()
        _cache[name] = (w, _device_int4(pk, w), _oracle_int4(oracle, w))
    return _cache[name]


def _u32(a):
    return np.ascontiguousarray(a).view(np.uint32)


def _decode(pk, w, dev, chunk_tokens, out_dtype):
    kc, vc, ks, vs = dev
    q = torch.from_numpy(w.q()).view(torch.bfloat16).cuda()
    bt = torch.from_numpy(w.block_tables).cuda()
    cl = torch.from_numpy(w.context_lens).cuda()
    mcl = max(w.max_context_len, 1)
    out = torch.empty(q.shape, dtype=out_dtype, device="cuda")
    nbytes = pk.kv8_decode_workspace_bytes(w.batch, w.num_q_heads, w.head_dim,
                                           mcl, chunk_tokens)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    pk.kv8_int4_paged_decode_attention(q, kc, vc, ks, vs, bt, cl, out, mcl,
                                       chunk_tokens=chunk_tokens, workspace=ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_int4_quantize_bit_exact(built, oracle_mod, name):
    w, dev, ref = _setup(built, oracle_mod, name)
    for g, o in zip(dev[:2], ref[:2]):
        assert np.array_equal(g.cpu().numpy(), o)
    for g, o in zip(dev[2:], ref[2:]):
        assert np.array_equal(_u32(g.cpu().numpy()), _u32(o))


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("chunk_tokens", [0, 64, 512])
@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_int4_decode_all_pairs(built, oracle_mod, name, chunk_tokens, out_dtype):
    w, dev, (kc, vc, ks, vs) = _setup(built, oracle_mod, name)
    ref = oracle_mod.decode_attention_int4(w.q(), kc, vc, ks, vs,
                                           w.block_tables, w.context_lens)
    dt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    gpu = _decode(built, w, dev, chunk_tokens, dt)
    U.assert_close(gpu, ref, bf16=(out_dtype == "bf16"))
    if out_dtype == "f32":
        assert np.abs(gpu - ref).max() < 1e-4


@pytest.fixture(scope="module")
def big_int4(built):
    _cache.clear()
    torch.cuda.empty_cache()
    w = W.llama8b_b64_32k()
    dev = _device_int4(built, w, itertools.chain(w.fill_segments(), [w.step_tokens()]))
    yield w, dev
    del dev
    torch.cuda.empty_cache()


BIG_SEQS = [0, 37, 63]


def test_big_int4_sampled_sequences(built, oracle_mod, big_int4):
    """The batch-64 x 32K workload in the bench's launch (chunk 512): the
    sampled sequences' packed codes and scales bit-exact against a private
    oracle cache of each, and their output rows within the decode
    tolerance."""
    w, dev = big_int4
    kc, vc, ks, vs = dev
    outs = {dt: _decode(built, w, dev, 512, dt) for dt in (torch.float32, torch.bfloat16)}
    for b in BIG_SEQS:
        t = int(w.context_lens[b])
        assert t % 16 == 0  # every page of the workload is full
        pkc, pvc, pks, pvs, table = U.oracle_int4_sequence(oracle_mod, w, b)
        blocks = torch.from_numpy(w.block_tables[b, :t // 16].astype(np.int64)).cuda()
        assert np.array_equal(kc[blocks].cpu().numpy(), pkc)
        assert np.array_equal(vc[blocks].cpu().numpy(), pvc)
        assert np.array_equal(_u32(ks[blocks].cpu().numpy()), _u32(pks))
        assert np.array_equal(_u32(vs[blocks].cpu().numpy()), _u32(pvs))
        ref = oracle_mod.decode_attention_int4(w.q()[b:b + 1], pkc, pvc, pks, pvs, table,
                                               w.context_lens[b:b + 1])[0]
        U.assert_close(outs[torch.float32][b], ref, bf16=False)
        U.assert_close(outs[torch.bfloat16][b], ref, bf16=True)
    assert all(np.all(np.isfinite(o)) for o in outs.values())
