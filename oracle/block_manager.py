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

- "为什么PagedAttention能让大模型推理吞吐量提升数倍", section "调度与抢占：当显存不够时
  怎么办", and "vLLM PagedAttention 深度解析" §5.2 (Swapping): a preempted
  request's KV blocks are moved out to CPU memory, which frees its GPU blocks,
  and are moved back into GPU blocks when it resumes; "LLM 推理引擎内部原理" §3.1
  lists the moves a scheduling step hands to the cache engine as block maps
  (blocks_to_swap_out / blocks_to_swap_in, next to blocks_to_copy).

Reading taken where the pages are silent: the copy-on-write check runs in
append_slot before the in-place write (vLLM's behaviour; page 3's listing has no
sharing and page 1 describes the copy only in prose), and `make_writable`
exposes the same check for an arbitrary logical block.

Swap readings (the pages give the idea, not the bookkeeping):
- CPU blocks form a second pool with its own FIFO free list and counts.
- swap_out(seqs) moves a whole set of sequences at once ("the whole request's
  blocks"). Every distinct GPU block they reference gets ONE new CPU block (a
  block shared by two of them is moved once), taken from the CPU free list in
  order of first appearance (sequences in the given order, each table in
  order). Each reference moves its count: the GPU block loses one per moved
  reference (freed at 0, so a block still used by a sequence left behind
  stays), the CPU block gains one. The result is the (gpu, cpu) block map.
- swap_in(seqs) is the mirror image, CPU -> GPU.
- Either is all or nothing: if the destination pool has fewer free blocks than
  the distinct blocks to move, nothing changes and the call returns None.
- A swapped-out sequence can be freed (its CPU blocks are released) or swapped
  in; appending to it, forking it or asking its table is an error.
"""
from __future__ import annotations

from collections import deque


class OutOfBlocks(Exception):
    pass


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None, num_cpu_blocks: int = 0,
                 cpu_free_order=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = range(self.num_blocks) if free_order is None else [int(b) for b in free_order]
        self.free = deque(order)
        self.ref = [0] * self.num_blocks
        self.tables: dict = {}
        self.lens: dict = {}
        self.num_cpu_blocks = int(num_cpu_blocks)
        corder = range(self.num_cpu_blocks) if cpu_free_order is None else [int(b) for b in cpu_free_order]
        self.cpu_free = deque(corder)
        self.cpu_ref = [0] * self.num_cpu_blocks
        self.swapped: set = set()

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

    def _resident(self, seq):
        if seq in self.swapped:
            raise ValueError(f"sequence {seq} is swapped out")

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
        self._resident(seq)
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
        self._resident(seq)
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
        self._resident(parent)
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def free_seq(self, seq):
        """Drop `seq`: every block's count falls by one; blocks at 0 return to
        the back of the free list, in table order (the CPU list for a swapped-out
        sequence)."""
        if seq in self.swapped:
            self.swapped.discard(seq)
            for c in self.tables.pop(seq, []):
                self.cpu_ref[c] -= 1
                if self.cpu_ref[c] == 0:
                    self.cpu_free.append(c)
        else:
            for b in self.tables.pop(seq, []):
                self._release(b)
        self.lens.pop(seq, None)

    # -- swapping ----------------------------------------------------------------
    def _move(self, seqs, src_ref, src_free, dst_ref, dst_free):
        """Moves the listed sequences' blocks from one pool to the other; returns
        the (src, dst) block map, or None (nothing changed) if dst lacks room."""
        distinct = []
        for s in seqs:
            for b in self.tables[s]:
                if b not in distinct:
                    distinct.append(b)
        if len(distinct) > len(dst_free):
            return None
        new_of = {}
        pairs = []
        for s in seqs:
            t = self.tables[s]
            for i, b in enumerate(t):
                if b not in new_of:
                    new_of[b] = dst_free.popleft()
                    dst_ref[new_of[b]] = 0
                    pairs.append((b, new_of[b]))
                dst_ref[new_of[b]] += 1
                src_ref[b] -= 1
                if src_ref[b] == 0:
                    src_free.append(b)
                t[i] = new_of[b]
        return pairs

    def swap_out(self, seqs):
        """GPU -> CPU for the listed (resident) sequences; the (gpu, cpu) map."""
        seqs = list(seqs)
        if any(s in self.swapped or s not in self.tables for s in seqs) or len(set(seqs)) != len(seqs):
            raise ValueError("swap_out takes distinct resident sequences")
        pairs = self._move(seqs, self.ref, self.free, self.cpu_ref, self.cpu_free)
        if pairs is not None:
            self.swapped.update(seqs)
        return pairs

    def swap_in(self, seqs):
        """CPU -> GPU for the listed swapped-out sequences; the (cpu, gpu) map."""
        seqs = list(seqs)
        if any(s not in self.swapped for s in seqs) or len(set(seqs)) != len(seqs):
            raise ValueError("swap_in takes distinct swapped-out sequences")
        pairs = self._move(seqs, self.cpu_ref, self.cpu_free, self.ref, self.free)
        if pairs is not None:
            self.swapped.difference_update(seqs)
        return pairs

    # -- views ---------------------------------------------------------------
    def block_table(self, seq):
        self._resident(seq)
        return list(self.tables[seq])

    def num_free(self) -> int:
        return len(self.free)
