"""Reference block manager -- TEST INFRASTRUCTURE ONLY.

A plain restatement of the host-side bookkeeping on the "PagedAttention" page
(shubhamtatvamasi):

* "The idea: page the KV cache" (the OS analogy table and the five-request
  figure): a sequence gets a new physical block from the free list only when
  its previous block is full; blocks come from anywhere.
* "Sharing and copy-on-write": one physical block may appear in several
  tables; every block counts its holders; a block that has filled up is not
  written again, so only a shared, partially filled last block is copied.
* "How does copy-on-write work for parallel sampling?": the samples' tables
  name the prompt's blocks, each counting its users; a sample that
  must append into a shared partial block takes a new block, has the tokens
  already there copied into it, drops its count on the old block and writes
  into the copy.

Free-list order is part of the input: ``free_order`` lists the physical ids in
the order they are handed out (front first); a freed block goes to the back.
The product's native block manager follows the same policy, and the tests
compare the two table for table.
"""
from __future__ import annotations

from collections import deque


class OutOfBlocks(RuntimeError):
    pass


class RefBlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = list(range(num_blocks)) if free_order is None else [int(x) for x in free_order]
        assert sorted(order) == list(range(num_blocks)), "free_order must be a permutation"
        self.free = deque(order)
        self.refcount = [0] * num_blocks
        self.tables = {}   # seq id -> list of physical ids
        self.lengths = {}  # seq id -> tokens held
        self.copies = []   # (src, dst) copy-on-write pairs, in order

    def _alloc(self) -> int:
        if not self.free:
            raise OutOfBlocks("free list is empty")
        blk = self.free.popleft()
        assert self.refcount[blk] == 0
        self.refcount[blk] = 1
        return blk

    def add_sequence(self, seq: int, num_tokens: int) -> None:
        """A new sequence holding num_tokens tokens: ceil(n / bs) fresh blocks."""
        assert seq not in self.tables
        n_blocks = -(-int(num_tokens) // self.block_size)
        self.tables[seq] = [self._alloc() for _ in range(n_blocks)]
        self.lengths[seq] = int(num_tokens)

    def fork(self, parent: int, child: int) -> None:
        """child shares every block of parent (each refcount + 1)."""
        assert child not in self.tables
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for blk in self.tables[child]:
            self.refcount[blk] += 1

    def append_slot(self, seq: int):
        """Reserve the slot of the next token of seq.

        Returns (slot, cow) where cow is None or the (src, dst) pair that the
        device must copy before the token is written."""
        table = self.tables[seq]
        pos = self.lengths[seq]
        bs = self.block_size
        cow = None
        if pos % bs == 0:
            # previous block full (or no block yet): take a fresh block now
            table.append(self._alloc())
        else:
            last = table[-1]
            if self.refcount[last] > 1:
                new = self._alloc()
                self.refcount[last] -= 1
                table[-1] = new
                cow = (last, new)
                self.copies.append(cow)
        slot = table[pos // bs] * bs + pos % bs
        self.lengths[seq] = pos + 1
        return slot, cow

    def free_sequence(self, seq: int) -> None:
        for blk in self.tables.pop(seq):
            self.refcount[blk] -= 1
            if self.refcount[blk] == 0:
                self.free.append(blk)
        del self.lengths[seq]

    def block_table(self, seq: int):
        return list(self.tables[seq])

    # -- invariants from "Sharing and copy-on-write" ------------------------
    def check_invariants(self) -> None:
        users = [0] * self.num_blocks
        for table in self.tables.values():
            for blk in table:
                users[blk] += 1
        assert users == self.refcount, "refcount != number of tables using the block"
        free = set(self.free)
        assert len(free) == len(self.free), "block listed twice in the free list"
        used = {b for b in range(self.num_blocks) if users[b] > 0}
        assert not (free & used), "a referenced block is on the free list"
        assert free | used == set(range(self.num_blocks)), "a block was lost"
        for seq, table in self.tables.items():
            need = -(-self.lengths[seq] // self.block_size)
            assert len(table) == need, "blocks held != ceil(len / block_size)"
