"""Host-side manager of the paged KV block pool.

The pool is a fixed set of physical blocks of ``block_size`` tokens.  Each
sequence owns a block table (logical block i -> physical block id).  Blocks
are handed out on demand and returned when a sequence ends
(chanyi.net.cn/article/49 section 三; lqnn.cn/news/235768 sections 3.2-3.3).
Sequences forked from a common prefix point at the same physical blocks,
counted by a reference count; the first append into a shared, partly filled
last block copies it first (copy-on-write, chanyi.net.cn/article/49 section 三).

Copy-on-write rule used here: an append copies the last block iff its
reference count is above one at that moment.  The last sharer to append
therefore writes in place.

The free list is a LIFO stack.  ``free_order`` fixes which blocks are handed
out first, so a seeded permutation scatters sequences across the pool.

Deferred reuse (``free_sequence(..., defer=True)``, then ``release_deferred()``):
the blocks of a sequence that ends after a decode step are held back until the
caller releases them, one step later.  A step's appends then never write a block
that the previous step's decode may still be reading, which lets the library
run those appends while that decode finishes (PA_APPEND_OVERLAP_PREVIOUS).
"""
from __future__ import annotations

import numpy as np


class OutOfBlocks(RuntimeError):
    """The pool has no free block left; the caller should queue the request."""


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int = 16, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = np.arange(num_blocks) if free_order is None else np.asarray(free_order)
        if sorted(order.tolist()) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of the pool")
        # pop() takes from the end, so the first block to hand out goes last.
        self._free: list[int] = [int(b) for b in order[::-1]]
        self.refcount = np.zeros(num_blocks, dtype=np.int64)
        self._deferred: list[int] = []  # freed, not yet back on the free list
        self.tables: dict[object, list[int]] = {}
        self.lens: dict[object, int] = {}

    # -- pool ---------------------------------------------------------------
    @property
    def num_free(self) -> int:
        return len(self._free)

    def _alloc(self) -> int:
        if not self._free:
            raise OutOfBlocks("KV block pool exhausted")
        b = self._free.pop()
        assert self.refcount[b] == 0
        self.refcount[b] = 1
        return b

    def _release(self, b: int) -> None:
        if self.refcount[b] <= 0:
            raise RuntimeError(f"double free of block {b}")
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            self._free.append(int(b))

    def blocks_needed(self, num_tokens: int) -> int:
        return -(-int(num_tokens) // self.block_size)

    # -- sequences ------------------------------------------------------------
    def add_sequence(self, seq_id, num_tokens: int) -> np.ndarray:
        """Allocate blocks for a new sequence of ``num_tokens`` tokens; return
        the slot (block * block_size + offset) of every token, in order.
        All-or-nothing: raises OutOfBlocks without side effects."""
        if seq_id in self.tables:
            raise KeyError(f"sequence {seq_id!r} exists")
        n = self.blocks_needed(num_tokens)
        if n > len(self._free):
            raise OutOfBlocks(f"need {n} blocks, {len(self._free)} free")
        table = [self._alloc() for _ in range(n)]
        self.tables[seq_id] = table
        self.lens[seq_id] = int(num_tokens)
        return self.slots(seq_id, 0, num_tokens)

    def fork(self, parent, child) -> None:
        """``child`` shares every block of ``parent`` (reference counts + 1)."""
        if child in self.tables:
            raise KeyError(f"sequence {child!r} exists")
        table = list(self.tables[parent])
        for b in table:
            self.refcount[b] += 1
        self.tables[child] = table
        self.lens[child] = self.lens[parent]

    def append_slot(self, seq_id):
        """Reserve the slot of the next token of ``seq_id``.

        Returns ``(slot, cow)``; ``cow`` is ``(src, dst)`` when the shared last
        block had to be copied first (the caller copies it on the device
        before writing the token), else None."""
        table = self.tables[seq_id]
        n = self.lens[seq_id]
        cow = None
        if n % self.block_size == 0:
            table.append(self._alloc())
        else:
            last = table[-1]
            if self.refcount[last] > 1:
                dst = self._alloc()
                self.refcount[last] -= 1
                table[-1] = dst
                cow = (int(last), int(dst))
        slot = table[n // self.block_size] * self.block_size + n % self.block_size
        self.lens[seq_id] = n + 1
        return int(slot), cow

    def free_sequence(self, seq_id, defer: bool = False) -> None:
        """Drop the sequence; with ``defer`` its blocks whose reference count falls
        to zero wait for release_deferred() before they can be handed out again."""
        for b in self.tables.pop(seq_id):
            if defer:
                if self.refcount[b] <= 0:
                    raise RuntimeError(f"double free of block {b}")
                self.refcount[b] -= 1
                if self.refcount[b] == 0:
                    self._deferred.append(int(b))
            else:
                self._release(b)
        del self.lens[seq_id]

    def release_deferred(self) -> None:
        """Put the blocks held back by free_sequence(defer=True) on the free list
        (in the order they were freed, as an immediate free would have)."""
        self._free.extend(self._deferred)
        self._deferred = []

    def slots(self, seq_id, start: int, stop: int) -> np.ndarray:
        table = np.asarray(self.tables[seq_id], dtype=np.int64)
        t = np.arange(start, stop, dtype=np.int64)
        return table[t // self.block_size] * self.block_size + t % self.block_size

    def block_table(self, seq_ids, max_blocks: int, pad: int = -1) -> np.ndarray:
        """int32 [len(seq_ids)][max_blocks]; entries past a sequence's last
        block hold ``pad`` and are never read by the decode kernels."""
        out = np.full((len(seq_ids), max_blocks), pad, dtype=np.int32)
        for i, s in enumerate(seq_ids):
            t = self.tables[s]
            if len(t) > max_blocks:
                raise ValueError(f"sequence {s!r} has {len(t)} blocks > {max_blocks}")
            out[i, : len(t)] = t
        return out

    # -- accounting ---------------------------------------------------------------
    def check_invariants(self) -> None:
        """Reference counts equal table references; free + used = pool; the
        free list holds each unused block exactly once."""
        refs = np.zeros(self.num_blocks, dtype=np.int64)
        for t in self.tables.values():
            for b in t:
                refs[b] += 1
        if not np.array_equal(refs, self.refcount):
            raise AssertionError("reference counts disagree with block tables")
        free = np.asarray(self._free + self._deferred, dtype=np.int64)
        if len(set(free.tolist())) != len(free):
            raise AssertionError("block on the free list twice")
        if np.any(self.refcount[free] != 0):
            raise AssertionError("free block still referenced")
        used = int(np.count_nonzero(self.refcount))
        if used + len(free) != self.num_blocks:
            raise AssertionError("free + used != pool")

    def used_blocks(self) -> int:
        return int(np.count_nonzero(self.refcount))
