"""The host block allocator (CPU): slots and block tables follow the paged
layout, whole full blocks are shared read-only with reference counts, a
sequence's new tokens always land in blocks it holds alone, and the tables
and slots it produces drive the oracle's cache to the same attention as a
private contiguous cache."""
import numpy as np
import pytest

import workloads as W
from paged_int8_kv_b200.blocks import BlockAllocator, OutOfBlocks

BS = 16


def test_slots_and_tables():
    a = BlockAllocator(8)
    a.add("x")
    s = a.append_slots("x", 20)
    blocks = a.blocks_of("x")
    assert len(blocks) == 2 and a.num_free == 6
    pos = np.arange(20)
    assert np.array_equal(s, np.asarray(blocks)[pos // BS] * BS + pos % BS)
    s2 = a.append_slots("x", 13)   # fills block 2's second... up to 33 tokens
    assert len(a.blocks_of("x")) == 3 and a.context_len("x") == 33
    assert np.array_equal(s2, np.asarray(a.blocks_of("x"))[np.arange(20, 33) // BS] * BS
                          + np.arange(20, 33) % BS)
    a.add("y")
    st = a.step_slots(["x", "y"])
    assert st[0] == a.blocks_of("x")[2] * BS + 1 and st[1] == a.blocks_of("y")[0] * BS
    bt = a.block_tables(["x", "y"])
    assert bt.shape == (2, 3) and bt.dtype == np.int32
    assert list(bt[0]) == a.blocks_of("x") and bt[1, 0] == a.blocks_of("y")[0]
    assert list(a.context_lens(["x", "y"])) == [34, 1]
    assert a.append_slots("y", 0).shape == (0,)
    with pytest.raises(ValueError):
        a.block_tables(["x"], max_blocks=2)


def test_fork_shares_full_blocks_read_only():
    a = BlockAllocator(16)
    a.add("p")
    a.append_slots("p", 40)                 # 2 full blocks + 8 tokens
    shared = a.fork("c", "p")               # shares the 2 full blocks
    assert shared == 32 and a.context_len("c") == 32
    pb = a.blocks_of("p")
    assert a.blocks_of("c") == pb[:2]
    assert [a.ref_count(b) for b in pb] == [2, 2, 1]
    # new tokens of either sequence never land in a shared block
    for seq, n in (("c", 5), ("p", 30), ("c", 20)):
        s = a.append_slots(seq, n)
        assert all(a.ref_count(int(x) // BS) == 1 for x in s)
    assert a.fork("d", "p", 17) == 16 and a.blocks_of("d") == pb[:1]
    with pytest.raises(ValueError):
        a.fork("e", "p", a.context_len("p") + 1)


def test_free_returns_blocks_when_last_holder_leaves():
    a = BlockAllocator(6)
    a.add("p")
    a.append_slots("p", 32)
    a.fork("c", "p")
    a.append_slots("c", 1)
    assert a.num_free == 3
    a.free("p")
    assert a.num_free == 3                  # the shared blocks stay with c
    a.free("c")
    assert a.num_free == 6 and "c" not in a


def test_out_of_blocks_changes_nothing():
    a = BlockAllocator(3)
    a.add("x")
    a.append_slots("x", 40)
    with pytest.raises(OutOfBlocks):
        a.append_slots("x", 20)             # needs 2 more, 0 free
    assert a.context_len("x") == 40 and a.num_free == 0
    assert a.append_slots("x", 8).shape == (8,)   # fits in the last block


def test_random_operations_keep_the_invariants():
    rng = np.random.default_rng(5)
    a = BlockAllocator(64)
    live = []
    owner = {}                               # slot -> sequence that wrote it
    for step in range(400):
        op = rng.integers(0, 10)
        if op < 2 or not live:
            name = f"s{step}"
            if live and op == 1:
                parent = live[rng.integers(len(live))]
                a.fork(name, parent, int(rng.integers(0, a.context_len(parent) + 1)))
            else:
                a.add(name)
            live.append(name)
        elif op < 8:
            seq = live[rng.integers(len(live))]
            try:
                s = a.append_slots(seq, int(rng.integers(0, 40)))
            except OutOfBlocks:
                continue
            for x in s:                      # a written slot is never handed out twice
                assert owner.get(int(x)) is None
                owner[int(x)] = seq
        else:
            seq = live.pop(rng.integers(len(live)))
            freed = set(a.blocks_of(seq))
            a.free(seq)
            for x in list(owner):
                if x // BS in freed and a.ref_count(x // BS) == 0:
                    del owner[x]
        # reference counts equal the tables listing each block
        refs = np.zeros(64, int)
        for s_ in live:
            for b in a.blocks_of(s_):
                refs[b] += 1
            assert len(a.blocks_of(s_)) == -(-a.context_len(s_) // BS)
        assert all(refs[b] == a.ref_count(b) for b in range(64))
        assert a.num_free == int((refs == 0).sum())


def test_allocator_drives_the_oracle_cache(oracle_mod):
    # two sequences sharing a 48-token prefix (3 whole blocks), one private;
    # K/V drawn per sequence; the oracle's attention over the allocator's
    # tables equals attention over private contiguous caches
    rng = np.random.default_rng(9)
    H, HQ, NB = 2, 8, 32
    a = BlockAllocator(NB)
    shape = (NB, H, BS, 128)
    kc, vc = np.full(shape, 127, np.int8), np.full(shape, 127, np.int8)
    ks, vs = np.full(shape[:3], np.nan, np.float32), np.full(shape[:3], np.nan, np.float32)

    def rows(n):
        return (W.f32_to_bf16_bits(rng.standard_normal((n, H, 128)).astype(np.float32)),
                W.f32_to_bf16_bits(rng.standard_normal((n, H, 128)).astype(np.float32)))

    def put(seq, k, v):
        s = a.append_slots(seq, k.shape[0])
        oracle_mod.quantize_append(k, s, kc, ks)
        oracle_mod.quantize_append(v, s, vc, vs)
    pk_, pv_ = rows(48)
    a.add("p")
    put("p", pk_, pv_)
    tails = {}
    for seq, n in (("p", 21), ("c", 37)):
        if seq == "c":
            assert a.fork("c", "p", 48) == 48
        tails[seq] = rows(n)
        put(seq, *tails[seq])
    a.add("solo")
    tails["solo"] = rows(29)
    put("solo", *tails["solo"])
    seqs = ["p", "c", "solo"]
    q = W.f32_to_bf16_bits(rng.standard_normal((3, HQ, 128)).astype(np.float32))
    out = oracle_mod.decode_attention(q, kc, vc, ks, vs, a.block_tables(seqs),
                                      a.context_lens(seqs))
    for i, seq in enumerate(seqs):
        k, v = tails[seq]
        if seq != "solo":
            k, v = np.concatenate([pk_, k]), np.concatenate([pv_, v])
        n = k.shape[0]
        nb = -(-n // BS)
        pc = np.full((nb, H, BS, 128), 127, np.int8), np.full((nb, H, BS, 128), 127, np.int8)
        ps = np.full((nb, H, BS), np.nan, np.float32), np.full((nb, H, BS), np.nan, np.float32)
        sl = np.arange(n, dtype=np.int64)
        oracle_mod.quantize_append(k, sl, pc[0], ps[0])
        oracle_mod.quantize_append(v, sl, pc[1], ps[1])
        ref = oracle_mod.decode_attention(q[i:i + 1], pc[0], pc[1], ps[0], ps[1],
                                          np.arange(nb, dtype=np.int32)[None, :],
                                          np.array([n], np.int32))
        assert np.array_equal(out[i], ref[0]), seq
