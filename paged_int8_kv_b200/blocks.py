"""Host-side block allocator for the paged cache.

Each sequence's tokens live in 16-token physical blocks that its block
table lists in logical order [KV Cache 优化全景解析——从基础原理到工程实践,
§4.2 PagedAttention: logical blocks map to physically scattered blocks
through a block table; blocks are allocated on demand; several sequences
may map the same physical block].  ``BlockAllocator`` hands out those blocks
and turns positions into the slot mapping (slot = block * 16 + offset) and
the block tables the append and decode calls take.

Sharing: ``fork`` lets a new sequence list a parent's whole, full blocks
(read-only, reference counted): the calls only ever write a sequence's own
blocks, because a sequence's new tokens always go to a block it holds alone
(a fork shares only full blocks, so its first new token opens a new block).
Copy-on-write of a partly filled shared block is not done here: a fork
shares floor(n / 16) blocks and the caller appends the remaining tokens.

Plain host bookkeeping (numpy); nothing here touches the GPU.
"""
from __future__ import annotations

import numpy as np


class OutOfBlocks(RuntimeError):
    pass


class BlockAllocator:
    def __init__(self, num_blocks: int, block_size: int = 16):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        # lowest block numbers first, so tables are easy to read in tests
        self._free = list(range(self.num_blocks - 1, -1, -1))
        self._refs = np.zeros(self.num_blocks, dtype=np.int64)
        self._tables: dict = {}   # seq id -> list of physical blocks
        self._lens: dict = {}     # seq id -> tokens held

    # ---------------------------------------------------------------- state
    @property
    def num_free(self) -> int:
        return len(self._free)

    def context_len(self, seq) -> int:
        return self._lens[seq]

    def blocks_of(self, seq) -> list:
        return list(self._tables[seq])

    def ref_count(self, block: int) -> int:
        return int(self._refs[block])

    def __contains__(self, seq) -> bool:
        return seq in self._tables

    # ------------------------------------------------------------ lifecycle
    def add(self, seq) -> None:
        if seq in self._tables:
            raise KeyError(f"sequence {seq!r} exists")
        self._tables[seq] = []
        self._lens[seq] = 0

    def fork(self, seq, parent, n_tokens: int | None = None) -> int:
        """A new sequence that shares the parent's first n_tokens (default:
        all of them) rounded down to whole blocks; returns the tokens shared.
        The caller appends the rest of its prefix itself."""
        if seq in self._tables:
            raise KeyError(f"sequence {seq!r} exists")
        plen = self._lens[parent]
        n = plen if n_tokens is None else int(n_tokens)
        if n < 0 or n > plen:
            raise ValueError(f"cannot share {n} of {plen} tokens")
        k = n // self.block_size
        shared = self._tables[parent][:k]
        for blk in shared:
            self._refs[blk] += 1
        self._tables[seq] = list(shared)
        self._lens[seq] = k * self.block_size
        return k * self.block_size

    def free(self, seq) -> None:
        """Drop a sequence; blocks no other sequence holds become free."""
        for blk in self._tables.pop(seq):
            self._refs[blk] -= 1
            if self._refs[blk] == 0:
                self._free.append(blk)
        del self._lens[seq]

    # ------------------------------------------------------------- appends
    def append_slots(self, seq, n: int) -> np.ndarray:
        """Reserve the next n positions of a sequence; returns their slots
        (int64 [n]).  Raises OutOfBlocks (and changes nothing) when the free
        blocks do not suffice."""
        n = int(n)
        if n < 0:
            raise ValueError("n must be >= 0")
        bs = self.block_size
        table = self._tables[seq]
        start = self._lens[seq]
        need = -(-(start + n) // bs) - len(table)
        if need > len(self._free):
            raise OutOfBlocks(f"{need} blocks needed, {len(self._free)} free")
        if start % bs and table and self._refs[table[-1]] > 1:
            # only full blocks are ever shared, so a partial last block is
            # always private
            raise AssertionError("partial block shared")
        for _ in range(max(need, 0)):
            blk = self._free.pop()
            self._refs[blk] = 1
            table.append(blk)
        pos = np.arange(start, start + n, dtype=np.int64)
        blocks = np.asarray(table, dtype=np.int64)
        self._lens[seq] = start + n
        if n == 0:
            return pos
        return blocks[pos // bs] * bs + pos % bs

    def step_slots(self, seqs) -> np.ndarray:
        """One new token for each sequence (a decode step); int64 [len(seqs)]."""
        return np.concatenate([self.append_slots(s, 1) for s in seqs]) if len(seqs) \
            else np.zeros(0, dtype=np.int64)

    # ------------------------------------------------------------- tables
    def block_tables(self, seqs, max_blocks: int | None = None,
                     pad: int = 0) -> np.ndarray:
        """int32 [len(seqs), max_blocks]: row b lists sequence seqs[b]'s blocks,
        padded with `pad` (never read: the calls read only the first
        ceil(len / block_size) entries of a row)."""
        rows = [self._tables[s] for s in seqs]
        width = max([len(r) for r in rows] + [1]) if max_blocks is None else int(max_blocks)
        out = np.full((len(rows), width), pad, dtype=np.int32)
        for i, r in enumerate(rows):
            if len(r) > width:
                raise ValueError(f"sequence {seqs[i]!r} holds {len(r)} blocks > {width}")
            out[i, :len(r)] = r
        return out

    def context_lens(self, seqs) -> np.ndarray:
        return np.asarray([self._lens[s] for s in seqs], dtype=np.int32)
