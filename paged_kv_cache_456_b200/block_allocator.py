"""Host-side KV block pool: a shuffled free list plus reference counts.

This is the bookkeeping half of paging, used here only to build the inputs
of the GPU path (block tables, slot mappings and copy-on-write pairs).

* The cache is cut into fixed-size blocks of ``block_size`` tokens (16 by
  default) and a per-sequence block table maps logical block ``j`` to a
  physical block id ("What vLLM Is and Why It Exists", section "The idea vLLM
  started from: pages"; skandtandon day-9 post, section "Idea 1:
  PagedAttention").
* A sequence of ``n`` tokens holds ``ceil(n / block_size)`` blocks, so it
  wastes at most ``block_size - 1`` token slots ("What vLLM Is and Why It
  Exists", sections "The idea vLLM started from: pages" and "Code"; "vLLM
  Solved the Wrong Bottleneck...", section "Paged Attention").
* Physical blocks may sit anywhere in the pool; the free list is a random
  permutation so consecutive logical blocks land on scattered physical ones
  (day-9 post, "Idea 1": a sequence's blocks need not be adjacent).
* Two sequences with a common prefix share physical blocks, and a shared block
  that must diverge is copied alone (copy-on-write) (day-9 post, "Idea 1",
  bullets "Sharing" and "Copy-on-write").  The pages name no reference count;
  sharing and copy-on-write imply one, so each block carries a count of the
  tables that point at it.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np


class OutOfBlocks(RuntimeError):
    """Raised when the pool has fewer free blocks than a request needs."""


def blocks_for_tokens(n_tokens: int, block_size: int = 16) -> int:
    """Blocks held by a sequence of ``n_tokens`` tokens: ceil(n / block_size)."""
    if n_tokens < 0:
        raise ValueError("n_tokens must be >= 0")
    return (n_tokens + block_size - 1) // block_size


class BlockAllocator:
    """Pool of ``num_blocks`` physical blocks of ``block_size`` token slots.

    ``rng`` (a ``numpy.random.Generator``) shuffles the free list once at
    construction; without it blocks are handed out in id order.  Block tables
    are plain Python lists of physical ids, owned by the caller.
    """

    def __init__(self, num_blocks: int, block_size: int = 16,
                 rng: Optional[np.random.Generator] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = rng.permutation(num_blocks) if rng is not None else np.arange(num_blocks)
        # pop() takes from the end, so reverse: the first block handed out is order[0]
        self._free: List[int] = [int(b) for b in order[::-1]]
        self.refcount = np.zeros(num_blocks, dtype=np.int64)
        # (src, dst) pairs produced by append_token's copy-on-write, for the caller to copy
        self.pending_copies: List[Tuple[int, int]] = []

    # -- queries -----------------------------------------------------------
    @property
    def num_free(self) -> int:
        return len(self._free)

    def blocks_for(self, n_tokens: int) -> int:
        return blocks_for_tokens(n_tokens, self.block_size)

    def slot_of(self, table: Sequence[int], token_index: int) -> int:
        """Flat slot id ``block * block_size + offset`` of a logical token."""
        j, off = divmod(token_index, self.block_size)
        return int(table[j]) * self.block_size + off

    # -- allocation --------------------------------------------------------
    def _pop(self) -> int:
        if not self._free:
            raise OutOfBlocks("no free KV blocks left in the pool")
        b = self._free.pop()
        assert self.refcount[b] == 0
        self.refcount[b] = 1
        return b

    def allocate(self, n_tokens: int) -> List[int]:
        """A fresh block table holding ``n_tokens`` tokens (all blocks private)."""
        need = self.blocks_for(n_tokens)
        if need > len(self._free):
            raise OutOfBlocks(f"need {need} blocks, {len(self._free)} free")
        return [self._pop() for _ in range(need)]

    def append_token(self, table: List[int], n_tokens: int) -> int:
        """Grow a sequence that holds ``n_tokens`` tokens by one token.

        A new block is taken only when the last one is full.  If the last
        block is shared, it is first made private by copy-on-write; the pair
        that must be copied is then returned in ``self.pending_copies``.
        Returns the slot id the new token is written to.
        """
        j, off = divmod(n_tokens, self.block_size)
        if off == 0:
            if j != len(table):
                raise ValueError("table length does not match n_tokens")
            table.append(self._pop())
        elif self.refcount[table[j]] > 1:
            pair = self.cow(table, j)
            if pair is not None:
                self.pending_copies.append(pair)
        return int(table[j]) * self.block_size + off

    # -- sharing -----------------------------------------------------------
    def fork(self, table: Sequence[int]) -> List[int]:
        """A second table sharing every block of ``table`` (refcounts + 1)."""
        for b in table:
            if self.refcount[b] <= 0:
                raise ValueError(f"block {b} is not allocated")
            self.refcount[b] += 1
        return list(table)

    def cow(self, table: List[int], logical_block: int) -> Optional[Tuple[int, int]]:
        """Make logical block ``logical_block`` of ``table`` private.

        If it is shared, a fresh block replaces it in ``table``, the old
        block's count drops by one, and ``(src, dst)`` is returned: the pair
        whose contents the device must copy.  A private block is left alone
        and ``None`` is returned.
        """
        old = int(table[logical_block])
        if self.refcount[old] <= 0:
            raise ValueError(f"block {old} is not allocated")
        if self.refcount[old] == 1:
            return None
        new = self._pop()
        self.refcount[old] -= 1
        table[logical_block] = new
        return (old, new)

    def free(self, table: Sequence[int]) -> None:
        """Drop one reference to each block of ``table``; return blocks at 0."""
        for b in table:
            if self.refcount[b] <= 0:
                raise ValueError(f"double free of block {b}")
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self._free.append(int(b))

    def check_conservation(self, tables: Sequence[Sequence[int]]) -> None:
        """Assert free + referenced = pool and counts equal table references."""
        counts = np.zeros(self.num_blocks, dtype=np.int64)
        for t in tables:
            for b in t:
                counts[b] += 1
        if not np.array_equal(counts, self.refcount):
            raise AssertionError("refcounts disagree with the tables")
        free = set(self._free)
        if len(free) != len(self._free):
            raise AssertionError("free list holds a block twice")
        used = set(np.nonzero(self.refcount)[0].tolist())
        if free & used or len(free) + len(used) != self.num_blocks:
            raise AssertionError("free list and referenced blocks do not partition the pool")


class ContiguousAllocator:
    """First-fit allocator over one linear range: the pre-paging baseline.

    Each request needs one contiguous run of units.  It exists to show
    external fragmentation: free memory split into gaps too small for a
    request even though the total would fit ("vLLM Solved the Wrong
    Bottleneck...", sections "Problem 2: Memory Fragmentation" and "Why
    transformers made it difficult").
    """

    def __init__(self, capacity: int):
        self.capacity = int(capacity)
        self.runs = {}  # name -> (start, length)

    def free_gaps(self) -> List[Tuple[int, int]]:
        taken = sorted(self.runs.values())
        gaps, pos = [], 0
        for start, length in taken:
            if start > pos:
                gaps.append((pos, start - pos))
            pos = start + length
        if pos < self.capacity:
            gaps.append((pos, self.capacity - pos))
        return gaps

    def allocate(self, name: str, length: int) -> int:
        for start, size in self.free_gaps():
            if size >= length:
                self.runs[name] = (start, length)
                return start
        raise OutOfBlocks(f"no contiguous run of {length} units")

    def free(self, name: str) -> None:
        del self.runs[name]

    @property
    def num_free(self) -> int:
        return sum(size for _, size in self.free_gaps())
