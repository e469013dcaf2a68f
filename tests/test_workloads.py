"""Host-side checks of the seeded workload generator (CPU only)."""
import math

import numpy as np

import workloads as W


def _check_layout(w: W.Workload):
    bs = w.block_size
    assert w.block_tables.dtype == np.int32 and w.context_lens.dtype == np.int32
    assert w.max_context_len <= w.max_blocks_per_seq * bs
    seen = {}
    for b, t in enumerate(w.context_lens):
        blocks = w.block_tables[b, :math.ceil(int(t) / bs)]
        assert np.all((blocks >= 0) & (blocks < w.num_blocks))
        for j, p in enumerate(blocks):
            seen.setdefault(int(p), set()).add((b, j))
    return seen


def test_tiny_layout():
    w = W.tiny()
    _check_layout(w)
    assert w.num_blocks == 64 and w.batch == 2
    assert list(w.context_lens) == [256, 200]
    assert len(w.poisoned_blocks()) == 64 - 16 - 13
    # table padding points at a poisoned block
    assert w.block_tables[1, 13] in set(w.poisoned_blocks().tolist())
    assert w.outlier_channels.shape == (2, 4)


def test_named_shapes():
    w = W.llama8b_b32()
    _check_layout(w)
    assert w.batch == 32 and w.group == 4
    assert w.context_lens.min() >= 1024 and w.context_lens.max() <= 4096
    assert w.outlier_channels.shape == (8, 3)
    w = W.llama8b_b64_32k()
    _check_layout(w)
    assert w.num_blocks == 64 * 2048 and w.max_context_len == 32768
    assert sorted(w.block_tables.reshape(-1).tolist()) == list(range(131072))
    w = W.pruned_compact()
    assert w.batch == 256 and set(w.context_lens.tolist()) == {544}
    assert all(len(p) == 544 and np.all(np.diff(p) > 0) for p in w.recorded_positions)
    w = W.prefix_shared_70b()
    seen = _check_layout(w)
    assert w.group == 8 and w.batch == 48
    shared = [p for p, users in seen.items() if len(users) > 1]
    assert len(shared) == 6 * 256
    assert all(len(seen[p]) == 8 for p in shared)


def test_fill_segments_cover_each_slot_once():
    for w in (W.tiny(), W.make_workload("t", 5, [33, 0, 16, 47], 4, 2,
                                        prefix_group=[-1, -1, 0, 0],
                                        prefix_len=0)):
        slots = []
        for k, v, s in w.fill_segments():
            assert k.shape == v.shape and k.shape[0] == s.shape[0]
            slots.append(s)
        ks, vs, ss = w.step_tokens()
        slots.append(ss[ss >= 0])
        allslots = np.concatenate(slots)
        assert len(np.unique(allslots)) == len(allslots)
        expect = sum(int(t) for t in w.context_lens)
        assert len(allslots) == expect


def test_prefix_segments_written_once():
    w = W.make_workload("p", 6, [48 + 5, 48 + 20, 48 + 1], 8, 1,
                        prefix_group=[0, 0, 0], prefix_len=48)
    segs = list(w.fill_segments())
    n = sum(s.shape[0] for _, _, s in segs) + 3
    assert n == 48 + 5 + 20 + 1
    # each sequence sees the prefix tokens then its own
    k0, _ = w.sequence_kv(0)
    k1, _ = w.sequence_kv(1)
    assert np.array_equal(k0[:48], k1[:48]) and k0.shape[0] == 53


def test_determinism():
    a, b = W.llama8b_b32(), W.llama8b_b32()
    assert np.array_equal(a.block_tables, b.block_tables)
    assert np.array_equal(a.q(), b.q())
    ka, va = a.private_kv(3)
    kb, vb = b.private_kv(3)
    assert np.array_equal(ka, kb) and np.array_equal(va, vb)


def test_bf16_rounding():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-3], dtype=np.float32)
    b = W.f32_to_bf16_bits(x)
    back = W.bf16_bits_to_f32(b)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: goes to the even one (1.0)
    assert back[1] == 1.0
    assert back[2] == np.float32(1.015625)
    assert back[0] == 1.0 and back[3] == -2.5


def _replay_kivi_calls(w):
    """Per sequence, the rows the KIVI fill and step calls append, keyed by
    position (every call's context_lens counts its rows: the new rows of
    sequence b sit at positions cl[b] - n_b .. cl[b] - 1)."""
    got = {b: {} for b in range(w.batch)}
    for k, v, cu, cl in list(w.kivi_fill_calls()) + [w.kivi_step_call()]:
        assert cu[0] == 0 and np.all(np.diff(cu) >= 0) and cu[-1] == k.shape[0]
        assert k.shape == v.shape and k.shape[1:] == (w.num_kv_heads, w.head_dim)
        for b in range(w.batch):
            n = int(cu[b + 1] - cu[b])
            assert 0 <= n <= int(cl[b])
            for i in range(n):
                pos = int(cl[b]) - n + i
                assert pos not in got[b], (b, pos)  # each position once
                got[b][pos] = (k[cu[b] + i], v[cu[b] + i])
    return got


def test_kivi_calls_append_every_position_once():
    w = W.make_workload("kv", 7, [33, 0, 16, 47, 1], 4, 2)
    got = _replay_kivi_calls(w)
    for b, t in enumerate(w.context_lens):
        assert sorted(got[b]) == list(range(int(t)))
        k, v = w.sequence_kv(b)
        for pos, (kr, vr) in got[b].items():
            assert np.array_equal(kr, k[pos]) and np.array_equal(vr, v[pos])


def test_kivi_calls_write_a_shared_prefix_once():
    w = W.make_workload("kp", 8, [48 + 5, 48 + 20, 48 + 1, 9], 8, 1,
                        prefix_group=[0, 0, 0, -1], prefix_len=48)
    got = _replay_kivi_calls(w)
    assert sorted(got[0]) == list(range(53))          # the first member: all
    assert sorted(got[1]) == list(range(48, 68))      # later members: suffix
    assert sorted(got[2]) == [48]
    assert sorted(got[3]) == list(range(9))
    # the step call appends exactly the last token of each sequence
    k, v, cu, cl = w.kivi_step_call()
    assert list(np.diff(cu)) == [1, 1, 1, 1] and list(cl) == [53, 68, 49, 9]
