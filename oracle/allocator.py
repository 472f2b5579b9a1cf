"""Block allocator with reference counts and per-sequence block tables (oracle).

TEST INFRASTRUCTURE ONLY.  An independent Python model of the host-side
allocator; the C++ allocator behind the C ABI must reproduce its state bit for
bit (tables, reference counts, free-pool contents and order) on the same trace.

Procedures (all from the pages' prose, cited by page title and section):

free pool / alloc
    Physical blocks are handed out from a free pool; a block whose reference
    count reaches zero is "returned to the free pool" ([SW] "Stop Wasting GPU
    Memory: A Deep Dive Into vLLM's PagedAttention", Technical Details, "Beam
    Search Optimization").  The pages fix no order; this model keeps the pool
    as a LIFO stack seeded from ``init_free_order`` (``alloc`` pops the last
    element, a freed block is pushed on top).

append (slot mapping)
    A sequence holding ``n`` tokens gets a new block exactly when its blocks
    are all full, i.e. when ``len(blocks) * B <= n`` (equivalently ``n % B ==
    0``) -- the allocation test of [ML] "49 vLLM / PagedAttention", "The block
    table (the paging idea)", read with the length counted *before* the append.
    The token goes to logical block ``n // B`` at offset ``n % B`` (the offset
    is left implicit in that listing) and the length then grows by one.

reference counts, fork, copy-on-write
    Branches that share a prefix point at the same physical blocks, each block
    carrying a reference count; on divergence only the diverging block is
    copied to a new physical block and the counts are adjusted ([SW] Technical
    Details, "Copy-on-Write for Parallel Sampling"; [PV] "PagedAttention: How
    Virtual Memory Paging Solved LLM KV Cache Waste", Key points, "Parallel
    sampling and copy-on-write").  Reading: a writer copies iff the block it
    writes into has a count above one at the moment it writes (the operating
    system rule the pages borrow); the source's count drops by one and the
    writer's table points at the copy.  Appending into a fresh block never
    copies.

free / prune
    Freeing a sequence decrements every block of its table, in table order;
    blocks reaching zero are pushed to the pool in that order ([SW] "Beam
    Search Optimization").

Errors leave the state unchanged: ``OutOfBlocks`` when the pool is empty,
``AllocatorStateError`` for a decrement below zero, sharing a free block or an
unknown sequence.
"""

from __future__ import annotations


class OutOfBlocks(RuntimeError):
    """The free pool is empty."""


class AllocatorStateError(RuntimeError):
    """A reference count would become invalid, or a sequence id is unknown."""


class BlockPool:
    """Free pool (LIFO stack) plus a reference count per physical block."""

    def __init__(self, num_blocks: int, init_free_order=None):
        if init_free_order is None:
            init_free_order = list(range(num_blocks - 1, -1, -1))
        order = [int(b) for b in init_free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("init_free_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.free = list(order)          # top of the stack is the last element
        self.refcount = [0] * num_blocks

    def alloc(self) -> int:
        if not self.free:
            raise OutOfBlocks("free pool is empty")
        b = self.free.pop()
        self.refcount[b] = 1
        return b

    def incref(self, blocks, by: int = 1) -> None:
        blocks = [int(b) for b in blocks]
        if by < 0:
            raise AllocatorStateError("negative increment")
        for b in blocks:
            if not 0 <= b < self.num_blocks or self.refcount[b] <= 0:
                raise AllocatorStateError(f"block {b} is not in use")
        for b in blocks:
            self.refcount[b] += by

    def decref(self, blocks) -> None:
        blocks = [int(b) for b in blocks]
        need = {}
        for b in blocks:
            if not 0 <= b < self.num_blocks:
                raise AllocatorStateError(f"block {b} outside the pool")
            need[b] = need.get(b, 0) + 1
        for b, c in need.items():
            if self.refcount[b] < c:
                raise AllocatorStateError(f"block {b} reference count would go below zero")
        for b in blocks:
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free.append(b)

    def cow(self, block: int):
        """Copy-on-write test for a block about to be written.

        Returns ``(target, copied)``: a fresh block and True when the block is
        shared (count > 1; its count drops by one), else the block itself and
        False.
        """
        block = int(block)
        if not 0 <= block < self.num_blocks or self.refcount[block] <= 0:
            raise AllocatorStateError(f"block {block} is not in use")
        if self.refcount[block] > 1:
            new = self.alloc()
            self.refcount[block] -= 1
            return new, True
        return block, False

    def num_free(self) -> int:
        return len(self.free)


class SequenceTables:
    """Per-sequence block tables and lengths on top of a ``BlockPool``."""

    def __init__(self, pool: BlockPool, block_size: int):
        self.pool = pool
        self.block_size = block_size
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self._next_id = 0

    def add(self) -> int:
        sid = self._next_id
        self._next_id += 1
        self.tables[sid] = []
        self.lens[sid] = 0
        return sid

    def _check(self, sid: int) -> None:
        if sid not in self.tables:
            raise AllocatorStateError(f"unknown sequence {sid}")

    def append(self, sid: int):
        """Place one new token; returns ``(slot, cow_pair or None)``."""
        self._check(sid)
        B = self.block_size
        n = self.lens[sid]
        blocks = self.tables[sid]
        pair = None
        if len(blocks) * B <= n:
            blocks.append(self.pool.alloc())
        else:
            last = blocks[-1]
            target, copied = self.pool.cow(last)
            if copied:
                blocks[-1] = target
                pair = (last, target)
        slot = blocks[n // B] * B + n % B
        self.lens[sid] = n + 1
        return slot, pair

    def append_many(self, sids):
        """One token for each listed sequence, in list order.

        Returns (slots, cow_pairs).  On running out of blocks the sequences
        already processed keep their tokens and the failing one is unchanged
        (the exception carries ``done`` = how many were placed).
        """
        slots, pairs = [], []
        for i, sid in enumerate(sids):
            try:
                slot, pair = self.append(int(sid))
            except OutOfBlocks as e:
                e.done = i
                raise
            slots.append(slot)
            if pair is not None:
                pairs.append(pair)
        return slots, pairs

    def fork(self, parent: int) -> int:
        """A child sharing every block of ``parent`` (each count grows by one)."""
        self._check(parent)
        self.pool.incref(self.tables[parent], 1)
        child = self.add()
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        return child

    def free(self, sid: int) -> None:
        self._check(sid)
        self.pool.decref(self.tables[sid])
        del self.tables[sid]
        del self.lens[sid]

    def table(self, sid: int) -> list[int]:
        self._check(sid)
        return list(self.tables[sid])
