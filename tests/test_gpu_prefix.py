"""kv8_paged_decode_attention_prefix on the GPU (through the C ABI).

Groups of sequences that share the blocks at the start of their block tables
are decoded with the shared pages read and scored once per group (on the
tcgen05 tensor cores, all the group's query rows together).  The shared
chunks' probabilities are rounded to fp16, as in extend attention, so the
bound is the decode tolerance |gpu - oracle| <= 2e-3 (plus half a bf16 ulp
for bf16 output) and not the 1e-4 the all-integer decode form keeps; the
mean error stays below 1e-4 (a misplaced row, key or head would not):
  * the prefix-shared workload (6 groups x 8 sequences, 4096-token prefix,
    64 q / 8 KV heads), every (sequence, head) against the oracle, fp32 and
    bf16 output, and against the plain call within 2e-3;
  * ragged cases: group sizes 1, 3, 8 and 11, a group of 20 members at 8
    query heads per KV head (two rounds of 16 members),
    sequences in no group, prefixes that are not a whole number of chunks,
    a member whose whole context is the prefix, every group size G;
  * a member shorter than its group's prefix sets bit 1 of the device
    status word (no fault, no hang).
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


def _prefix_decode(pk, cache, q, bt, cl, w, groups, plens, chunk, out_dtype):
    pg = torch.from_numpy(np.asarray(groups, dtype=np.int32)).cuda()
    pl = torch.from_numpy(np.asarray(plens, dtype=np.int32)).cuda()
    sizes = np.bincount(np.asarray([g for g in groups if g >= 0], dtype=np.int64),
                        minlength=len(plens)) if len(plens) else np.zeros(0)
    out = torch.full(q.shape, float("nan"), dtype=out_dtype, device="cuda")
    ws = cache.workspace(w.batch, w.num_q_heads, w.max_context_len, chunk)
    pk.kv8_paged_decode_attention_prefix(
        q, cache.k_cache, cache.v_cache, cache.k_scales, cache.v_scales, bt,
        cl, out, w.max_context_len, pg, pl,
        int(sizes.max()) if len(sizes) else 0,
        int(max(plens)) if len(plens) else 0, chunk_tokens=chunk, workspace=ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("chunk", [256, 512])
def test_prefix_shared_workload(pk, oracle_mod, chunk):
    w = W.prefix_shared_70b()
    cache, q, bt, cl = U.device_inputs(w)
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    ref = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    groups = w.prefix_group.tolist()
    plens = [w.prefix_len] * (max(groups) + 1)
    for dt, bf in ((torch.float32, False), (torch.bfloat16, True)):
        got = _prefix_decode(pk, cache, q, bt, cl, w, groups, plens, chunk, dt)
        U.assert_close(got, ref, bf16=bf)
        if not bf:
            assert np.abs(got - ref).mean() < 1e-4
            plain = U.gpu_decode(cache, q, bt, cl, w, chunk_tokens=chunk)
            assert np.abs(got - plain).max() <= 2e-3


@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 4), (8, 2), (16, 2)])
def test_prefix_ragged_groups(pk, oracle_mod, hq, hkv):
    # group 0: 3 members, prefix 200 tokens (with 64-token chunks 3 whole
    # chunks are shared and 8 tokens stay with each member); group 1: 11
    # members (two rounds of 8), prefix 128, one member's whole context is the
    # prefix; group 2: 1 member; sequences 1, 16 and 17 in no group
    grp = [0, -1, 0, 0] + [1] * 11 + [2, -1, -1]
    suffix = [40, 300, 1, 77, 0, 15, 16, 17, 64, 65, 3, 100, 1, 2, 33, 500, 10, 90]
    plen_of = {0: 200, 1: 128, 2: 256}
    lens = [(plen_of[g] if g >= 0 else 0) + s for g, s in zip(grp, suffix)]
    first = {g: grp.index(g) for g in plen_of}
    w = W.make_workload("pfx", 6100 + hq + hkv, lens, hq, hkv, extra_blocks=8,
                        chunk_tokens=64)
    # members list their group's first member's blocks for the prefix; a
    # block only partly inside the prefix (group 0's block 12: tokens
    # 192..207) stays private, holding the shared tokens 192..199 too
    bt = w.block_tables.copy()
    for g, plen in plen_of.items():
        for b, x in enumerate(grp):
            if x == g and b != first[g]:
                bt[b, :plen // 16] = bt[first[g], :plen // 16]
    w.block_tables = bt
    base = w.private_kv

    def kv(b, _base=base):
        k, v = _base(b)
        g = grp[b]
        if g >= 0 and b != first[g]:
            k0, v0 = _base(first[g])
            n = plen_of[g]
            k = np.concatenate([k0[:n], k[n:]])
            v = np.concatenate([v0[:n], v[n:]])
        return k, v
    w.private_kv = kv
    cache, q, btd, cl = U.device_inputs(w)
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    ref = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    plens = [plen_of[0], plen_of[1], plen_of[2]]
    for chunk in (64, 128):
        got = _prefix_decode(pk, cache, q, btd, cl, w, grp, plens, chunk,
                             torch.float32)
        U.assert_close(got, ref, bf16=False)
        assert np.abs(got - ref).mean() < 1e-4


def test_prefix_two_rounds(pk, oracle_mod):
    # 20 members at G = 8: rows of 16 members per item, so two rounds
    grp = [0] * 20 + [-1]
    plen = 128
    lens = [plen + s for s in range(5, 105, 5)] + [70]
    w = W.make_workload("pfx2", 6300, lens, 16, 2, extra_blocks=4,
                        chunk_tokens=64)
    bt = w.block_tables.copy()
    for b in range(1, 20):
        bt[b, :plen // 16] = bt[0, :plen // 16]
    w.block_tables = bt
    base = w.private_kv

    def kv(b, _base=base):
        k, v = _base(b)
        if 0 < b < 20:
            k0, v0 = _base(0)
            k = np.concatenate([k0[:plen], k[plen:]])
            v = np.concatenate([v0[:plen], v[plen:]])
        return k, v
    w.private_kv = kv
    cache, q, btd, cl = U.device_inputs(w)
    kc, vc, ks, vs = U.oracle_full_cache(oracle_mod, w)
    ref = oracle_mod.decode_attention(w.q(), kc, vc, ks, vs, w.block_tables,
                                      w.context_lens)
    got = _prefix_decode(pk, cache, q, btd, cl, w, grp, [plen], 64,
                         torch.float32)
    U.assert_close(got, ref, bf16=False)
    assert np.abs(got - ref).mean() < 1e-4


def test_prefix_member_shorter_than_prefix_sets_status(pk):
    lens = [300, 300, 100]  # member 2 is shorter than the 256-token prefix
    w = W.make_workload("pfxbad", 6200, lens, 8, 2, extra_blocks=2)
    bt = w.block_tables.copy()
    bt[1, :16] = bt[0, :16]
    bt[2, :7] = bt[0, :7]
    w.block_tables = bt
    cache, q, btd, cl = U.device_inputs(w)
    assert pk.kv8_read_device_status(clear=True) == 0
    _prefix_decode(pk, cache, q, btd, cl, w, [0, 0, 0], [256], 128,
                   torch.float32)
    assert pk.kv8_read_device_status(clear=True) == 2
