"""GPU parity of the KIVI cache variant against the CPU oracle.

  * kv8_kivi_append: every full page's codes, scales and zero points (keys
    per channel, values per token), unpacked from the library's page record,
    equal the oracle's bit for bit (zero points by value: +0 and -0 are the
    same minimum); every sequence's tail rows equal the oracle's;
  * the same cache however the tokens are split into append calls (one call
    per sequence, then one token at a time, then the step);
  * kv8_kivi_paged_decode_attention: every (sequence, query head) against the
    oracle's fp64 attention (full pages dequantised, the partial page from the
    tail), within the decode tolerance (2e-3, plus half a bf16 ulp for bf16
    output) and within 1e-4 for fp32 output; groups of 1, 2, 4 and 8 query
    heads, split (64, 512) and unsplit, ragged and empty contexts, shared
    prefixes, permuted block tables.
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

REC = 2176  # KV8_KIVI_PAGE_BYTES


@pytest.fixture(scope="module")
def pk():
    from paged_int8_kv_b200 import build
    build.build()
    import paged_int8_kv_b200 as m
    assert m.KV8_KIVI_PAGE_BYTES == REC
    yield m
    assert m.kv8_read_device_status(clear=True) == 0


def _ragged(group, seed=2100):
    return W.make_workload(f"kivi_ragged_g{group}", seed + group,
                           [1, 15, 16, 17, 0, 300, 1000, 33, 48, 511], 4 * group, 4,
                           extra_blocks=5, outliers=(3, 10.0))


CASES = {
    "tiny": W.tiny,
    "llama8b_b32": W.llama8b_b32,
    "pruned_compact": W.pruned_compact,
    "ragged_g1": lambda: _ragged(1),
    "ragged_g2": lambda: _ragged(2),
    "ragged_g4": lambda: _ragged(4),
    "ragged_g8": lambda: _ragged(8),
    "prefix_shared_70b": W.prefix_shared_70b,
}


def unpack_records(rec: np.ndarray):
    """The page records (uint8 [NB, H, 2176]) in the oracle's plain layout."""
    def words(lo, hi, dt):
        return np.ascontiguousarray(rec[..., lo:hi]).view(dt)
    shifts = (2 * np.arange(16, dtype=np.uint32))[:, None]
    kw, vw = words(0, 512, np.uint32), words(512, 1024, np.uint32)
    kc = ((kw[..., None, :] >> shifts) & 3).astype(np.uint8)  # [NB, H, 16, 128]
    vc = ((vw[..., None, :] >> shifts) & 3).astype(np.uint8)
    return (kc, words(1024, 1536, np.float32), words(1536, 2048, np.float32),
            vc, words(2048, 2112, np.float32), words(2112, 2176, np.float32))


def _dev(a, bf16=False):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.view(torch.bfloat16) if bf16 else t


def device_kivi(pk, w, calls):
    cache = torch.zeros((w.num_blocks, w.num_kv_heads, REC), dtype=torch.uint8,
                        device="cuda")
    tail = torch.full((w.batch, w.num_kv_heads, 2, 16, 128), -1,
                      dtype=torch.int16, device="cuda").view(torch.bfloat16)
    bt = _dev(w.block_tables)
    for k, v, cu, cl in calls:
        pk.kv8_kivi_append(_dev(k, True), _dev(v, True), _dev(cu), _dev(cl), bt,
                           cache, tail, max(int(np.diff(cu).max(initial=0)), 1))
    torch.cuda.synchronize()
    return cache, tail


def oracle_kivi(oracle, w, calls):
    c = oracle.KiviCache(w.num_blocks, w.num_kv_heads, w.batch)
    for k, v, cu, cl in calls:
        oracle.kivi_append(c, k, v, cu, cl, w.block_tables)
    return c


def _calls(w):
    return list(w.kivi_fill_calls()) + [w.kivi_step_call()]


_cache = {}


def _setup(pk, oracle, name):
    if name not in _cache:
        _cache.clear()  # one workload (and its reference) at a time
        torch.cuda.empty_cache()
        w = CASES[name]()
        calls = _calls(w)
        _cache[name] = (w, device_kivi(pk, w, calls), oracle_kivi(oracle, w, calls))
    return _cache[name]


def full_page_blocks(w):
    return np.unique(np.concatenate(
        [w.block_tables[b, :int(t) // 16] for b, t in enumerate(w.context_lens)]
        + [np.zeros(0, np.int32)])).astype(np.int64)


def assert_same_fields(got, ref):
    """Unpacked records against the oracle's fields: codes and scales bit
    for bit, zero points by value."""
    names = ("k codes", "k scales", "k zeros", "v codes", "v scales", "v zeros")
    for name, g, r in zip(names, got, ref):
        if name.endswith("zeros"):
            assert np.array_equal(g, r), name           # by value
        elif g.dtype == np.float32:
            assert np.array_equal(g.view(np.uint32), r.view(np.uint32)), name
        else:
            assert np.array_equal(g, r), name


def assert_same_cache(w, dev, oc):
    cache, tail = dev
    blocks = full_page_blocks(w)
    got = unpack_records(cache.cpu().numpy()[blocks])
    assert_same_fields(got, [a[blocks] for a in oc.fields()])
    t = tail.view(torch.int16).cpu().numpy().view(np.uint16)
    for b, n in enumerate(w.context_lens):
        f = int(n) % 16
        assert np.array_equal(t[b, :, :, :f], oc.tail[b, :, :, :f]), b


@pytest.mark.parametrize("name", list(CASES))
def test_kivi_append_bit_exact(pk, oracle_mod, name):
    w, dev, oc = _setup(pk, oracle_mod, name)
    assert_same_cache(w, dev, oc)


def test_kivi_append_split_calls(pk, oracle_mod):
    # the last 40 tokens of every sequence one call at a time
    w = _ragged(4, seed=2300)
    rows = [w.sequence_kv(b) for b in range(w.batch)]
    lens = w.context_lens.astype(np.int64)
    first = np.maximum(lens - 40, 0)
    calls = []
    cu = np.zeros(w.batch + 1, np.int32)
    cu[1:] = np.cumsum(first)
    calls.append((np.concatenate([rows[b][0][:first[b]] for b in range(w.batch)]),
                  np.concatenate([rows[b][1][:first[b]] for b in range(w.batch)]),
                  cu, first.astype(np.int32)))
    cur = first.copy()
    while (cur < lens).any():
        has = cur < lens
        ks = [rows[b][0][cur[b]:cur[b] + 1] for b in range(w.batch) if has[b]]
        vs = [rows[b][1][cur[b]:cur[b] + 1] for b in range(w.batch) if has[b]]
        cu = np.concatenate([[0], np.cumsum(has)]).astype(np.int32)
        cur = cur + has
        calls.append((np.concatenate(ks), np.concatenate(vs), cu, cur.astype(np.int32)))
    dev = device_kivi(pk, w, calls)
    oc = oracle_kivi(oracle_mod, w, _calls(w))  # the same tokens in two calls
    assert_same_cache(w, dev, oc)


def _decode(pk, w, dev, chunk, out_dtype):
    cache, tail = dev
    q = _dev(w.q(), True)
    mcl = max(w.max_context_len, 1)
    out = torch.empty(q.shape, dtype=out_dtype, device="cuda")
    nbytes = pk.kv8_decode_workspace_bytes(w.batch, w.num_q_heads, w.head_dim,
                                           mcl, chunk)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    pk.kv8_kivi_paged_decode_attention(q, cache, tail, _dev(w.block_tables),
                                       _dev(w.context_lens), out, mcl,
                                       chunk_tokens=chunk, workspace=ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("chunk", [0, 64, 512])
@pytest.mark.parametrize("name", list(CASES))  # slowest: one setup per case
def test_kivi_decode_all_pairs(pk, oracle_mod, name, chunk, out_dtype):
    w, dev, oc = _setup(pk, oracle_mod, name)
    if ("ref", name) not in _cache:
        _cache[("ref", name)] = oracle_mod.kivi_decode_attention(
            w.q(), oc, w.block_tables, w.context_lens)
    ref = _cache[("ref", name)]
    dt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    gpu = _decode(pk, w, dev, chunk, dt)
    U.assert_close(gpu, ref, bf16=(out_dtype == "bf16"))
    if out_dtype == "f32":
        assert np.abs(gpu - ref).max() < 1e-4


@pytest.fixture(scope="module")
def big_kivi(pk):
    _cache.clear()
    torch.cuda.empty_cache()
    w = W.llama8b_b64_32k()
    dev = device_kivi(pk, w, itertools.chain(w.kivi_fill_calls(), [w.kivi_step_call()]))
    yield w, dev
    del dev
    torch.cuda.empty_cache()


BIG_SEQS = [0, 37, 63]


def test_big_kivi_sampled_sequences(pk, oracle_mod, big_kivi):
    """The batch-64 x 32K workload, filled and decoded as the bench does
    (one append call per sequence, the step's token, chunk 512): the sampled
    sequences' page records bit-exact against a private oracle cache of each,
    and their output rows within the decode tolerance."""
    w, dev = big_kivi
    cache, tail = dev
    outs = {dt: _decode(pk, w, dev, 512, dt) for dt in (torch.float32, torch.bfloat16)}
    for b in BIG_SEQS:
        t = int(w.context_lens[b])
        oc, table = U.oracle_kivi_sequence(oracle_mod, w, b)
        blocks = torch.from_numpy(w.block_tables[b, :t // 16].astype(np.int64)).cuda()
        assert_same_fields(unpack_records(cache[blocks].cpu().numpy()),
                           [a[:t // 16] for a in oc.fields()])
        ref = oracle_mod.kivi_decode_attention(w.q()[b:b + 1], oc, table,
                                               w.context_lens[b:b + 1])[0]
        U.assert_close(outs[torch.float32][b], ref, bf16=False)
        U.assert_close(outs[torch.bfloat16][b], ref, bf16=True)
    assert all(np.all(np.isfinite(o)) for o in outs.values())


def test_kivi_rejects_bad_shapes(pk):
    w = W.tiny()
    cache = torch.zeros((w.num_blocks, w.num_kv_heads, REC), dtype=torch.uint8, device="cuda")
    tail = torch.zeros((w.batch, w.num_kv_heads, 2, 16, 128), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((w.batch, 6, 128), dtype=torch.bfloat16, device="cuda")  # group 3
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    with pytest.raises(pk.Kv8Error):
        pk.kv8_kivi_paged_decode_attention(q, cache, tail, _dev(w.block_tables),
                                           _dev(w.context_lens), out,
                                           w.max_context_len, chunk_tokens=0)
    q = torch.zeros((w.batch, 8, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    with pytest.raises(pk.Kv8Error):  # split without a workspace
        pk.kv8_kivi_paged_decode_attention(q, cache, tail, _dev(w.block_tables),
                                           _dev(w.context_lens), out,
                                           w.max_context_len, chunk_tokens=64)
