"""Oracle block manager: free list, block tables, slot mapping, ref counts, CoW.

TEST INFRASTRUCTURE (see oracle/__init__.py). Plain Python, written for
readability, not speed.

What it follows:
- "LLM 推理引擎内部原理" §2.3 (Block 分配器): the free pool is a FIFO of block
  ids (taken from the front, returned to the back); a new request takes
  ceil(n_tokens / block_size) blocks; appending a token writes into the last
  block while it has room (slot = last_block * block_size + len % block_size)
  and otherwise takes one new block from the front of the free list (slot =
  new_block * block_size); an empty free list is out-of-memory (None).
- "vLLM PagedAttention 解析" §4.1 (Parallel Sampling / Copy-on-Write): forked
  samples map their logical blocks to the same physical blocks and raise the
  blocks' reference counts; the first write into a shared block (ref > 1)
  copies it to a fresh block for the writer, whose table then points at the
  copy, and both counts drop back (old block ref - 1, new block ref 1).
- "vLLM PagedAttention 解析" §4.2 (Beam Search): a block whose reference count
  reaches 0 goes back to the free pool at once.

Reading taken where the pages are silent: the copy-on-write check runs in
append_slot before the in-place write (vLLM's behaviour; page 3's listing has no
sharing and page 1 describes the copy only in prose), and `make_writable`
exposes the same check for an arbitrary logical block.
"""
from __future__ import annotations

from collections import deque


class OutOfBlocks(Exception):
    pass


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = range(self.num_blocks) if free_order is None else [int(b) for b in free_order]
        self.free = deque(order)
        self.ref = [0] * self.num_blocks
        self.tables: dict = {}
        self.lens: dict = {}

    # -- helpers ---------------------------------------------------------------
    def _take(self):
        if not self.free:
            return None
        b = self.free.popleft()
        self.ref[b] = 1
        return b

    def _release(self, b: int):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def slot(self, seq, pos: int) -> int:
        """Slot of logical token position `pos` of `seq`: block table lookup,
        then in-block offset."""
        t = self.tables[seq]
        return t[pos // self.block_size] * self.block_size + pos % self.block_size

    # -- the block engine's calls ------------------------------------------
    def allocate(self, seq, num_tokens: int):
        """New request of num_tokens prompt tokens: ceil(n / block_size) blocks.
        Returns the slot of each prompt token, or None (nothing taken) when the
        pool cannot hold it."""
        n_blk = -(-int(num_tokens) // self.block_size)
        if n_blk > len(self.free):
            return None
        self.tables[seq] = [self._take() for _ in range(n_blk)]
        self.lens[seq] = int(num_tokens)
        return [self.slot(seq, p) for p in range(num_tokens)]

    def append_slot(self, seq):
        """Slot for the next token of `seq`, as (slot, copy) where copy is a
        (src, dst) block pair when a shared last block had to be copied first,
        else None. Returns None when the free list is empty (out of memory)."""
        n = self.lens[seq]
        t = self.tables[seq]
        copy = None
        if n % self.block_size != 0:
            last = t[-1]
            if self.ref[last] > 1:
                new = self._take()
                if new is None:
                    return None
                self.ref[last] -= 1
                t[-1] = new
                copy = (last, new)
        else:
            new = self._take()
            if new is None:
                return None
            t.append(new)
        self.lens[seq] = n + 1
        return self.slot(seq, n), copy

    def make_writable(self, seq, logical_block: int):
        """Copy-on-write of one logical block: if its physical block is shared,
        give `seq` a private copy. Returns the (src, dst) pair to copy, or None
        when the block was already private. Raises OutOfBlocks if no block is free."""
        t = self.tables[seq]
        old = t[logical_block]
        if self.ref[old] <= 1:
            return None
        new = self._take()
        if new is None:
            raise OutOfBlocks()
        self.ref[old] -= 1
        t[logical_block] = new
        return (old, new)

    def fork(self, parent, child):
        """`child` shares all of `parent`'s physical blocks (ref + 1 each)."""
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def free_seq(self, seq):
        """Drop `seq`: every block's count falls by one; blocks at 0 return to
        the back of the free list, in table order."""
        for b in self.tables.pop(seq, []):
            self._release(b)
        self.lens.pop(seq, None)

    # -- views ---------------------------------------------------------------
    def block_table(self, seq):
        return list(self.tables[seq])

    def num_free(self) -> int:
        return len(self.free)
