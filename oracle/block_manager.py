"""Plain-Python model of the host block allocator (oracle side).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows [P2] "vLLM推理引擎架构：PagedAttention机制与高吞吐推理" §2.2
"Block管理器实现": a Python list of free block ids; ``allocate(n)`` fails
with an out-of-memory error when fewer than n ids are free and otherwise
takes the first n; ``free(ids)`` appends the ids to the back of the list.
Shared-prefix blocks carry a reference count ([P4] "大模型推理KV Cache内存管理
与PagedAttention分页显存实战": several sampling requests of one prompt share
the prefix blocks, whose lifetime a reference count manages): ``share``
increments it and a block goes back to the free list only when ``free``
brings it to zero. The page does not say what the initial free-list order
is; it starts as ``list(range(num_blocks))`` there, and a caller may pass a
permutation instead (a seeded shuffle is an input, not part of the method).
"""
from __future__ import annotations


class OutOfBlocks(Exception):
    pass


class BlockManager:
    def __init__(self, num_blocks: int, initial_free_order=None):
        self.num_blocks = num_blocks
        if initial_free_order is None:
            self.free_blocks = list(range(num_blocks))
        else:
            order = [int(b) for b in initial_free_order]
            if sorted(order) != list(range(num_blocks)):
                raise ValueError("initial order must be a permutation of range(num_blocks)")
            self.free_blocks = order
        self.refcount = [0] * num_blocks

    def allocate(self, n: int) -> list:
        if n < 0:
            raise ValueError("negative count")
        if len(self.free_blocks) < n:
            raise OutOfBlocks(f"Need {n} blocks, only {len(self.free_blocks)} available")
        taken = self.free_blocks[:n]
        self.free_blocks = self.free_blocks[n:]
        for b in taken:
            self.refcount[b] = 1
        return taken

    def share(self, block_id: int) -> None:
        if not (0 <= block_id < self.num_blocks) or self.refcount[block_id] == 0:
            raise ValueError("share of a free or unknown block")
        self.refcount[block_id] += 1

    def free(self, block_ids) -> None:
        ids = [int(b) for b in block_ids]
        # validate the whole request first: nothing changes on error
        drops = {}
        for b in ids:
            if not (0 <= b < self.num_blocks):
                raise ValueError("free of an unknown block")
            drops[b] = drops.get(b, 0) + 1
            if drops[b] > self.refcount[b]:
                raise ValueError("free of a free block (refcount underflow)")
        for b in ids:
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free_blocks.append(b)

    def copy_on_write(self, block_id: int):
        """Make ``block_id`` private to the holder that is about to write into it.

        [P4] lets several block tables reference one physical block, with a
        reference count for its lifetime, but says nothing about writing into
        such a block. The reading taken here: a holder that must write into a
        block with refcount > 1 first takes a fresh block (allocated like any
        other: the head of the free list), moves its reference there and
        copies the contents; a block with refcount 1 is written in place.
        Returns ``(block_to_write, must_copy)``; on OutOfBlocks nothing changes.
        """
        b = int(block_id)
        if not (0 <= b < self.num_blocks) or self.refcount[b] == 0:
            raise ValueError("copy_on_write of a free or unknown block")
        if self.refcount[b] == 1:
            return b, False
        (new,) = self.allocate(1)
        self.refcount[b] -= 1
        return new, True

    def num_free(self) -> int:
        return len(self.free_blocks)
