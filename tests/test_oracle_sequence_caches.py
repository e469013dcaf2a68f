"""The private one-sequence oracle caches the full-size GPU tests compare
against (CPU): a sequence's private KIVI / INT4 cache holds the same pages
as the whole batch's oracle cache, and its attention rows equal the batch's
bit for bit (the oracle's arithmetic does not depend on block numbering or
on the other sequences)."""
import numpy as np

import workloads as W
from tests import gpu_util as U


def _batch():
    return W.make_workload("seqcache", 3100, [47, 16, 0, 33, 1], 8, 2,
                           extra_blocks=4, outliers=(3, 10.0))


def test_kivi_private_cache_matches_the_batch(oracle_mod):
    w = _batch()
    full = oracle_mod.KiviCache(w.num_blocks, w.num_kv_heads, w.batch)
    for call in list(w.kivi_fill_calls()) + [w.kivi_step_call()]:
        oracle_mod.kivi_append(full, *call, w.block_tables)
    ref = oracle_mod.kivi_decode_attention(w.q(), full, w.block_tables, w.context_lens)
    for b, t in enumerate(int(x) for x in w.context_lens):
        c, table = U.oracle_kivi_sequence(oracle_mod, w, b)
        for a_full, a_seq in zip(full.fields(), c.fields()):
            got = a_seq[:t // 16]
            want = a_full[w.block_tables[b, :t // 16]]
            assert np.array_equal(got.view(np.uint8), want.view(np.uint8))
        assert np.array_equal(c.tail[0, :, :, :t % 16], full.tail[b, :, :, :t % 16])
        out = oracle_mod.kivi_decode_attention(w.q()[b:b + 1], c, table,
                                               w.context_lens[b:b + 1])
        assert np.array_equal(out[0], ref[b])


def test_int4_private_cache_matches_the_batch(oracle_mod):
    w = _batch()
    shape = (w.num_blocks, w.num_kv_heads, 16, 64)
    kc, vc = np.zeros(shape, np.uint8), np.zeros(shape, np.uint8)
    ks, vs = np.zeros(shape[:3], np.float32), np.zeros(shape[:3], np.float32)
    for k, v, s in list(w.fill_segments()) + [w.step_tokens()]:
        oracle_mod.quantize_append_int4(k, s, kc, ks)
        oracle_mod.quantize_append_int4(v, s, vc, vs)
    ref = oracle_mod.decode_attention_int4(w.q(), kc, vc, ks, vs, w.block_tables,
                                           w.context_lens)
    for b, t in enumerate(int(x) for x in w.context_lens):
        pk, pv, pks, pvs, table = U.oracle_int4_sequence(oracle_mod, w, b)
        pages = (t + 15) // 16
        blocks = w.block_tables[b, :pages]
        for r in range(t):  # every written row of the sequence
            j, o = r // 16, r % 16
            assert np.array_equal(pk[j, :, o], kc[blocks[j], :, o])
            assert np.array_equal(pv[j, :, o], vc[blocks[j], :, o])
            assert np.array_equal(pks[j, :, o], ks[blocks[j], :, o])
        out = oracle_mod.decode_attention_int4(w.q()[b:b + 1], pk, pv, pks, pvs, table,
                                               w.context_lens[b:b + 1])
        assert np.array_equal(out[0], ref[b])
