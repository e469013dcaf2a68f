"""Seeded synthetic inputs for paged INT8 KV decode attention.

This module is shared by the tests, the smoke check and the bench, and feeds
both the CUDA path and the CPU oracle.  It holds no arithmetic of the method
(no quantisation, no attention): it only draws random bf16 tensors, context
lengths and block placements, and lays them out as the caller will hand them
to either side.

Recipe (the same for every workload):
  * RNG: numpy ``default_rng`` (PCG64) seeded with a list ``[seed, stream, i]``
    so that every stream can be drawn on its own and in parallel:
      stream 0 -> layout (block permutation, context lengths, outlier
                  channels, pruned positions),
      stream 1 -> K and V of sequence i's private tokens (K first, then V),
      stream 2 -> K and V of shared-prefix group i,
      stream 3 -> q.
  * Values: fp32 ``standard_normal`` rounded to bf16 (round to nearest even).
  * K outlier channels: the same channels for every token of a KV head,
    multiplied by a fixed factor before rounding.
  * Physical blocks: a seeded permutation of ``num_blocks`` ids handed out
    to sequences in order; blocks no sequence uses stay "poisoned".
  * Poison: unused cache bytes hold code 127 and unused scales hold NaN, so a
    read of an unused slot shows up in the output.

The five named workloads follow the shapes quoted for the method: a tiny GQA-4
case, the Llama-3.1-8B layer shape at batch 32 and at batch 64 x 32K, a pruned
544-token compact layout at batch 256, and a LLaMA-3-70B-shaped batch whose
groups of 8 sequences share a 4096-token prefix.
"""
from __future__ import annotations

import math
from collections import deque
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

POISON_CODE = 127
HEAD_DIM = 128
BLOCK_SIZE = 16


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, stream: int, i: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream), int(i)])


@dataclass
class Workload:
    """One decode batch over a paged cache, plus how to fill that cache."""
    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    context_lens: np.ndarray            # int32 [B]
    block_tables: np.ndarray            # int32 [B, max_blocks_per_seq]
    num_blocks: int
    head_dim: int = HEAD_DIM
    block_size: int = BLOCK_SIZE
    chunk_tokens: int = 512
    outlier_channels: np.ndarray | None = None   # int [H_kv, n] or None
    outlier_factor: float = 1.0
    # shared prefix: group id per sequence (-1 = none) and tokens per prefix
    prefix_group: np.ndarray | None = None
    prefix_len: int = 0
    recorded_positions: list | None = None       # pruned layout only; unused
    description: str = ""
    _q: np.ndarray | None = field(default=None, repr=False)

    # ----------------------------------------------------------- shapes
    @property
    def batch(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.batch else 0

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def used_blocks(self) -> np.ndarray:
        """Distinct physical blocks referenced by any sequence."""
        ids = [self.block_tables[b, :math.ceil(int(t) / self.block_size)]
               for b, t in enumerate(self.context_lens)]
        if not ids:
            return np.zeros(0, dtype=np.int64)
        return np.unique(np.concatenate(ids).astype(np.int64))

    def poisoned_blocks(self) -> np.ndarray:
        used = np.zeros(self.num_blocks, dtype=bool)
        used[self.used_blocks()] = True
        return np.nonzero(~used)[0]

    # ----------------------------------------------------------- values
    def q(self) -> np.ndarray:
        """bf16 bits [B, H_q, D]."""
        if self._q is None:
            g = _rng(self.seed, 3)
            x = g.standard_normal((self.batch, self.num_q_heads, self.head_dim),
                                  dtype=np.float32)
            self._q = f32_to_bf16_bits(x)
        return self._q

    def _draw_kv(self, g: np.random.Generator, n: int):
        shape = (n, self.num_kv_heads, self.head_dim)
        k = g.standard_normal(shape, dtype=np.float32)
        if self.outlier_channels is not None and n:
            for h in range(self.num_kv_heads):
                k[:, h, self.outlier_channels[h]] *= np.float32(self.outlier_factor)
        v = g.standard_normal(shape, dtype=np.float32)
        return f32_to_bf16_bits(k), f32_to_bf16_bits(v)

    def _private_start(self, b: int) -> int:
        if self.prefix_group is not None and self.prefix_group[b] >= 0:
            return self.prefix_len
        return 0

    def prefix_kv(self, grp: int):
        return self._draw_kv(_rng(self.seed, 2, grp), self.prefix_len)

    def private_kv(self, b: int):
        """K, V bf16 bits of sequence b's private tokens (positions start..T_b)."""
        n = int(self.context_lens[b]) - self._private_start(b)
        return self._draw_kv(_rng(self.seed, 1, b), max(n, 0))

    def sequence_kv(self, b: int):
        """K, V bf16 bits [T_b, H_kv, D] of every token sequence b attends to."""
        k, v = self.private_kv(b)
        if self._private_start(b):
            pk, pv = self.prefix_kv(int(self.prefix_group[b]))
            k = np.concatenate([pk, k], axis=0)
            v = np.concatenate([pv, v], axis=0)
        return k, v

    def slots(self, b: int, positions: np.ndarray) -> np.ndarray:
        pos = np.asarray(positions, dtype=np.int64)
        blk = self.block_tables[b, pos // self.block_size].astype(np.int64)
        return blk * self.block_size + pos % self.block_size

    # ----------------------------------------------------------- cache fill
    def fill_segments(self, include_last: bool = False, threads: int = 8):
        """Yield (k, v, slot_mapping) covering every used slot exactly once.

        By default the last token of each sequence is left out: it is the
        token a decode step appends (see ``step_tokens``).  Segments are
        produced by a thread pool, one sequence (or prefix group) each.
        """
        jobs = []
        if self.prefix_group is not None:
            for grp in sorted(set(int(x) for x in self.prefix_group if x >= 0)):
                b0 = int(np.nonzero(self.prefix_group == grp)[0][0])
                jobs.append(("prefix", grp, b0))
        for b in range(self.batch):
            jobs.append(("private", b, b))

        def work(job):
            kind, i, b = job
            if kind == "prefix":
                k, v = self.prefix_kv(i)
                pos = np.arange(self.prefix_len)
            else:
                k, v = self.private_kv(i)
                start = self._private_start(i)
                pos = np.arange(start, start + k.shape[0])
                if not include_last and k.shape[0]:
                    k, v, pos = k[:-1], v[:-1], pos[:-1]
            return k, v, self.slots(b, pos)

        with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
            for seg in ex.map(work, jobs):
                if seg[2].shape[0]:
                    yield seg

    def step_tokens(self):
        """The decode step's new tokens: K, V [B, H_kv, D] and slots [B].

        Token b is position T_b - 1 of sequence b (slot -1 when T_b == 0).
        """
        B = self.batch
        k = np.zeros((B, self.num_kv_heads, self.head_dim), dtype=np.uint16)
        v = np.zeros_like(k)
        slots = np.full(B, -1, dtype=np.int64)
        for b in range(B):
            t = int(self.context_lens[b])
            if t == 0 or t <= self._private_start(b):
                continue
            kb, vb = self.private_kv(b)
            k[b], v[b] = kb[-1], vb[-1]
            slots[b] = self.slots(b, [t - 1])[0]
        return k, v, slots

    # ----------------------------------------------------------- KIVI fill
    def kivi_fill_calls(self, threads: int = 8):
        """Append calls that put every token but each sequence's last into a
        KIVI cache, one call per sequence: yields (k, v, cu_new [B+1],
        context_lens [B]) with only sequence b's rows, in sequence order.  A
        shared prefix is appended by its group's first member only (its
        blocks are shared; the prefix is a whole number of pages), the other
        members start after it.  Up to ``threads`` sequences are drawn ahead
        on a thread pool, so host memory holds that many sequences' rows."""
        B = self.batch
        seen = set()
        jobs = []
        for b in range(B):
            n = max(int(self.context_lens[b]) - 1, 0)
            lo = 0
            if self.prefix_group is not None and self.prefix_group[b] >= 0:
                grp = int(self.prefix_group[b])
                lo = self.prefix_len if grp in seen else 0
                seen.add(grp)
            lo = min(lo, n)
            if n > lo:
                jobs.append((b, lo, n))

        def work(job):
            b, lo, n = job
            k, v = self.sequence_kv(b)
            cu = np.zeros(B + 1, np.int32)
            cu[b + 1:] = n - lo
            cl = np.zeros(B, np.int32)
            cl[b] = n
            return k[lo:n], v[lo:n], cu, cl

        ahead = max(1, threads)
        with ThreadPoolExecutor(max_workers=ahead) as ex:
            pending = deque(ex.submit(work, j) for j in jobs[:ahead])
            nxt = ahead
            while pending:
                res = pending.popleft().result()
                if nxt < len(jobs):
                    pending.append(ex.submit(work, jobs[nxt]))
                    nxt += 1
                yield res

    def kivi_step_call(self):
        """The decode step's append call: each sequence's last token
        (sequences with an empty context append nothing)."""
        k, v, slots = self.step_tokens()
        has = slots >= 0
        cu = np.concatenate([[0], np.cumsum(has)]).astype(np.int32)
        return k[has], v[has], cu, self.context_lens.astype(np.int32)

    # ----------------------------------------------------------- accounting
    def token_heads(self) -> int:
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads

    def unique_token_heads(self) -> int:
        return int(self.used_blocks().shape[0]) * self.block_size * self.num_kv_heads


# ------------------------------------------------------------------ builders
def _assign_blocks(perm: np.ndarray, context_lens, block_size, mbs,
                   pad_block: int, prefix_group=None, prefix_blocks=0):
    B = len(context_lens)
    tables = np.full((B, max(mbs, 1)), pad_block, dtype=np.int32)
    cursor = 0
    group_blocks = {}
    for b in range(B):
        nblk = math.ceil(int(context_lens[b]) / block_size)
        start = 0
        if prefix_group is not None and prefix_group[b] >= 0:
            grp = int(prefix_group[b])
            if grp not in group_blocks:
                group_blocks[grp] = perm[cursor:cursor + prefix_blocks]
                cursor += prefix_blocks
            tables[b, :prefix_blocks] = group_blocks[grp]
            start = prefix_blocks
        n = nblk - start
        tables[b, start:nblk] = perm[cursor:cursor + n]
        cursor += n
    return tables, cursor


def make_workload(name: str, seed: int, context_lens, num_q_heads: int,
                  num_kv_heads: int, *, extra_blocks: int = 0,
                  outliers: tuple[int, float] | None = None,
                  prefix_group=None, prefix_len: int = 0,
                  chunk_tokens: int = 512, num_blocks: int | None = None,
                  description: str = "") -> Workload:
    """General builder: lengths given, blocks shuffled, optional sharing."""
    cl = np.asarray(context_lens, dtype=np.int32)
    bs = BLOCK_SIZE
    g0 = _rng(seed, 0)
    pg = None if prefix_group is None else np.asarray(prefix_group, dtype=np.int32)
    prefix_blocks = prefix_len // bs
    assert prefix_len % bs == 0
    need = 0
    seen = set()
    for b in range(len(cl)):
        nblk = math.ceil(int(cl[b]) / bs)
        if pg is not None and pg[b] >= 0:
            assert int(cl[b]) > prefix_len
            if int(pg[b]) not in seen:
                seen.add(int(pg[b]))
                need += prefix_blocks
            nblk -= prefix_blocks
        need += nblk
    nb = num_blocks if num_blocks is not None else need + extra_blocks
    assert nb >= need
    perm = g0.permutation(nb).astype(np.int32)
    mbs = max([math.ceil(int(t) / bs) for t in cl] + [1])
    # table padding points at a block no sequence uses, when there is one
    pad = int(perm[need]) if nb > need else 0
    tables, used = _assign_blocks(perm, cl, bs, mbs, pad, pg, prefix_blocks)
    oc = None
    factor = 1.0
    if outliers is not None:
        n_ch, factor = outliers
        oc = np.stack([np.sort(g0.choice(HEAD_DIM, n_ch, replace=False))
                       for _ in range(num_kv_heads)])
    return Workload(name=name, seed=seed, num_q_heads=num_q_heads,
                    num_kv_heads=num_kv_heads, context_lens=cl,
                    block_tables=tables, num_blocks=nb,
                    chunk_tokens=chunk_tokens, outlier_channels=oc,
                    outlier_factor=factor, prefix_group=pg,
                    prefix_len=prefix_len, description=description)


def tiny() -> Workload:
    """Batch 2, lengths {256, 200}, 8 q / 2 KV heads, 64 shuffled blocks,
    4 outlier K channels x8 per KV head."""
    return make_workload("tiny_gqa4_b2", 1001, [256, 200], 8, 2, num_blocks=64,
                         outliers=(4, 8.0),
                         description="batch 2, context {256,200}, 8q/2kv heads, "
                                     "64 shuffled physical blocks (35 poisoned)")


def llama8b_b32() -> Workload:
    """Llama-3.1-8B layer shape, batch 32, lengths uniform in [1024, 4096],
    ceil(2% of 128) = 3 outlier K channels x10 per KV head."""
    g = _rng(1002, 0, 1)
    cl = g.integers(1024, 4096, size=32, endpoint=True)
    return make_workload("llama8b_b32_ctx1k-4k", 1002, cl, 32, 8,
                         outliers=(3, 10.0),
                         description="batch 32, context U[1024,4096], 32q/8kv")


def llama8b_b64_32k() -> Workload:
    """Llama-3.1-8B layer shape, batch 64, every context 32768 tokens,
    131072 shuffled blocks (4 GiB of codes), split-K over 512 tokens."""
    return make_workload("llama8b_b64_ctx32k", 1003, [32768] * 64, 32, 8,
                         description="batch 64, context 32768, 32q/8kv, chunk 512")


def pruned_compact() -> Workload:
    """Batch 256 sequences each holding a 544-token retained budget drawn as
    sorted random positions from original lengths in [2048, 16384]."""
    w = make_workload("pruned_b256_ctx544", 1004, [544] * 256, 32, 8,
                      description="batch 256, 544 retained tokens each, 32q/8kv")
    g = _rng(1004, 0, 1)
    orig = g.integers(2048, 16384, size=256, endpoint=True)
    w.recorded_positions = [np.sort(g.choice(int(n), 544, replace=False))
                            for n in orig]
    return w


def prefix_shared_70b() -> Workload:
    """LLaMA-3-70B layer shape (64 q / 8 KV heads), batch 48 in 6 groups of 8
    sharing a 4096-token prefix, private suffixes of 64..1024 tokens."""
    g = _rng(1005, 0, 1)
    suffix = g.integers(64, 1024, size=48, endpoint=True)
    grp = np.repeat(np.arange(6), 8)
    return make_workload("prefix_shared_70b_b48", 1005, 4096 + suffix, 64, 8,
                         prefix_group=grp, prefix_len=4096,
                         description="batch 48 = 6 groups x 8 sharing a 4096-token "
                                     "prefix, suffix U[64,1024], 64q/8kv")


NAMED = {
    "tiny": tiny,
    "llama8b_b32": llama8b_b32,
    "llama8b_b64_32k": llama8b_b64_32k,
    "pruned_compact": pruned_compact,
    "prefix_shared_70b": prefix_shared_70b,
}
