"""Host logic of the context-parallel decode (CPU only): shard bounds,
per-rank table views, and the all-gather layout the merge expects, the last
on world-size-2 gloo ranks."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

from paged_int8_kv_b200 import context_parallel as CP  # noqa: E402


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_bounds_cover_the_context(world):
    for n in [0, 1, 15, 16, 511, 512, 513, 1000, 4096, 32768, 32769]:
        for ct in (16, 64, 512):
            spans = [CP.shard_bounds(n, world, r, ct) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (s0, e0), (s1, e1) in zip(spans, spans[1:]):
                assert e0 == s1 and s0 <= e0
            for s, e in spans:
                assert e == s or s % ct == 0  # parts start on chunk boundaries
            sizes = [-(-(e - s) // ct) for s, e in spans]
            assert max(sizes) - min(sizes) <= 1  # chunks spread evenly


def test_local_tables_slice_the_global_tables():
    rng = np.random.default_rng(3)
    lens = np.array([1000, 16, 0, 513], dtype=np.int32)
    bt = rng.permutation(400)[:4 * 63].reshape(4, 63).astype(np.int32)
    for world in (1, 2, 3):
        seen = [[] for _ in lens]
        for r in range(world):
            t, ll, mx = CP.local_tables(bt, lens, world, r, 64)
            # the same bound and table width on every rank, covering its part
            assert mx == CP.max_local_len(lens, world, 64) >= ll.max()
            assert t.shape[1] == max(-(-mx // 16), 1)
            for b in range(len(lens)):
                s, e = CP.shard_bounds(int(lens[b]), world, r, 64)
                assert ll[b] == e - s
                nblk = -(-(e - s) // 16)
                assert list(t[b, :nblk]) == list(bt[b, s // 16:s // 16 + nblk])
                seen[b] += list(range(s, e))
        for b, n in enumerate(lens):
            assert seen[b] == list(range(int(n)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = torch.full((48,), rank + 1, dtype=torch.uint8)
        mine[0] = 100 + rank
        allp = CP.gather_partials(mine, world)
        q.put((rank, allp.numpy().copy()))
    finally:
        dist.destroy_process_group()


def test_gather_layout_is_rank_major_on_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        a = res[rank]
        for r in range(world):
            blk = a[r * 48:(r + 1) * 48]
            assert blk[0] == 100 + r and np.all(blk[1:] == r + 1)
