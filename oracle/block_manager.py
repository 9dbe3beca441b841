"""Plain-Python model of the paged KV-cache block manager -- TEST INFRASTRUCTURE.

It states the allocation rules directly, with no optimisation, so tests can compare the
product's C++ block manager against it bit for bit (block tables, slots, copy-on-write pairs,
reference counts and free-list order).

Rules, from "Memory Optimization in LLM Serving with PagedAttention":
  * section "How PagedAttention Works": the KV memory is a pool of equal fixed-size blocks;
    a sequence is a run of logical blocks, each mapped through its block table to some
    physical block; physical blocks are taken only when generation needs them (on-demand
    allocation), so only a sequence's last block is ever partly empty.
  * section "Advanced Capabilities: Memory Sharing with Copy-on-Write": parallel samples map
    their prompt blocks to the same physical blocks (a fork bumps each block's reference
    count); before a sequence appends a token into a shared block it checks the block's
    reference count, and if it is above one it takes a fresh block, copies the old block's
    content there, repoints its own table entry, and only then writes.
And from "vLLM and PagedAttention: How Ideas from Operating Systems Accelerated LLM
Inference": 16-token blocks by default; memory is allocated as generation proceeds; when
memory runs short, whole sequences are evicted by swapping them to CPU
memory.  Modelled here as a second, host pool of blocks: swapping a sequence out gives each of
its blocks a fresh host block (the device block loses one reference and is freed when none is
left), swapping it in gives each host block a fresh device block; a swapped-out sequence can
only be swapped in or freed.

Readings where the pages are silent:
  * the free list is first-in first-out: allocation pops its head, a freed block joins its
    tail; its initial order is given by the caller (default 0 .. num_blocks-1);
  * a block whose reference count drops to zero is freed, in the order of the freeing
    sequence's table;
  * a failed allocation (empty free list) raises ``OutOfBlocks`` and changes nothing; a batch
    of appends is all or nothing.
"""
import copy
from collections import deque


class OutOfBlocks(RuntimeError):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks, block_size=16, free_order=None):
        if num_blocks < 0 or block_size < 1:
            raise ValueError("bad pool shape")
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free order must be a permutation of the blocks")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = deque(order)
        self.ref = [0] * num_blocks
        self.tables = {}
        self.lens = {}
        self.swapped = set()
        self.host_free = deque()
        self.num_host_blocks = 0

    def set_host_pool(self, num_host_blocks, free_order=None):
        order = list(range(num_host_blocks)) if free_order is None else \
            [int(b) for b in free_order]
        if sorted(order) != list(range(num_host_blocks)):
            raise ValueError("host free order must be a permutation")
        if self.swapped:
            raise ValueError("sequences are swapped out")
        self.num_host_blocks = num_host_blocks
        self.host_free = deque(order)

    # -- queries --------------------------------------------------------------------
    def num_free(self):
        return len(self.free)

    def refcount(self, blk):
        return self.ref[blk]

    def block_table(self, seq):
        return list(self.tables[seq])

    def seq_len(self, seq):
        return self.lens[seq]

    def free_order(self):
        return list(self.free)

    def host_free_order(self):
        return list(self.host_free)

    def is_swapped(self, seq):
        if seq not in self.tables:
            raise KeyError(seq)
        return seq in self.swapped

    def waste(self, seq):
        """Empty slots in the sequence's own blocks (internal fragmentation)."""
        return len(self.tables[seq]) * self.block_size - self.lens[seq]

    # -- operations -----------------------------------------------------------------
    def _take(self):
        if not self.free:
            raise OutOfBlocks("no free block")
        blk = self.free.popleft()
        assert self.ref[blk] == 0
        self.ref[blk] = 1
        return blk

    def add_seq(self, seq, num_tokens):
        """Register a sequence whose first ``num_tokens`` tokens need slots (a prompt)."""
        if seq in self.tables:
            raise KeyError("sequence exists")
        if num_tokens < 0:
            raise ValueError("negative length")
        need = -(-num_tokens // self.block_size)
        if need > len(self.free):
            raise OutOfBlocks("prompt needs %d blocks, %d free" % (need, len(self.free)))
        self.tables[seq] = [self._take() for _ in range(need)]
        self.lens[seq] = num_tokens

    def append_slot(self, seq):
        """Give the next token of ``seq`` a slot; returns (slot, cow) with cow = (src, dst)
        when a shared last block had to be copied first, else None."""
        if seq in self.swapped:
            raise ValueError("sequence is swapped out")
        table = self.tables[seq]
        n = self.lens[seq]
        B = self.block_size
        cow = None
        if n % B == 0:
            table.append(self._take())
        else:
            last = table[-1]
            if self.ref[last] > 1:
                dst = self._take()
                self.ref[last] -= 1
                table[-1] = dst
                cow = (last, dst)
        slot = table[n // B] * B + n % B
        self.lens[seq] = n + 1
        return slot, cow

    def append_slots(self, seqs):
        """Append one token to each sequence in order; all or nothing.
        Returns (slots, cow_pairs)."""
        if any(s in self.swapped for s in seqs):
            raise ValueError("sequence is swapped out")
        saved = (copy.copy(self.free), list(self.ref),
                 {s: list(t) for s, t in self.tables.items()}, dict(self.lens))
        slots, pairs = [], []
        try:
            for s in seqs:
                slot, cow = self.append_slot(s)
                slots.append(slot)
                if cow is not None:
                    pairs.append(cow)
        except OutOfBlocks:
            self.free, self.ref, self.tables, self.lens = saved
            raise
        return slots, pairs

    def fork(self, parent, child):
        """``child`` maps the same physical blocks as ``parent`` (shared pages)."""
        if child in self.tables:
            raise KeyError("child exists")
        if parent in self.swapped:
            raise ValueError("parent is swapped out")
        table = self.tables[parent]
        for blk in table:
            self.ref[blk] += 1
        self.tables[child] = list(table)
        self.lens[child] = self.lens[parent]

    def free_seq(self, seq):
        """Drop a finished sequence; blocks nobody else maps go back to the free list."""
        if seq in self.swapped:
            self.swapped.discard(seq)
            self.host_free.extend(self.tables.pop(seq))
        else:
            for blk in self.tables.pop(seq):
                self.ref[blk] -= 1
                if self.ref[blk] == 0:
                    self.free.append(blk)
        del self.lens[seq]

    def swap_out(self, seq):
        """Move ``seq`` to host blocks.  Returns [(device_block, host_block), ...] in table
        order: the copies the caller must make before any freed device block is reused."""
        if seq in self.swapped:
            raise ValueError("already swapped out")
        table = self.tables[seq]
        if len(table) > len(self.host_free):
            raise OutOfBlocks("host pool exhausted")
        pairs = []
        for j, blk in enumerate(table):
            h = self.host_free.popleft()
            pairs.append((blk, h))
            self.ref[blk] -= 1
            if self.ref[blk] == 0:
                self.free.append(blk)
            table[j] = h
        self.swapped.add(seq)
        return pairs

    def swap_in(self, seq):
        """Move ``seq`` back to fresh device blocks.  Returns [(host_block, device_block)]."""
        if seq not in self.swapped:
            raise ValueError("not swapped out")
        table = self.tables[seq]
        if len(table) > len(self.free):
            raise OutOfBlocks("no free block")
        pairs = []
        for j, h in enumerate(table):
            blk = self._take()
            pairs.append((h, blk))
            self.host_free.append(h)
            table[j] = blk
        self.swapped.discard(seq)
        return pairs
