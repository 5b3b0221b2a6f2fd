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

Prefix caching ([P4] "Prefix Caching": KV blocks of a shared prompt prefix
are reused across requests and found by hash matching) keeps a map from
block content hash to block, with the policy of ``acquire_prefix``.
"""
from __future__ import annotations


import hashlib

import numpy as np


class OutOfBlocks(Exception):
    pass


def block_hash(parent, tokens) -> bytes:
    """Content hash of one full block for prefix caching ([P4], Prefix
    Caching: shareable prefix blocks are found by hash matching; the page
    names no hash). SHA-256 of the parent block's 32-byte hash (32 zero bytes
    for a prompt's first block) followed by the token ids as little-endian
    int32 (hashlib's SHA-256 is the library step)."""
    head = bytes(32) if parent is None else bytes(parent)
    assert len(head) == 32
    return hashlib.sha256(head + np.asarray(tokens, dtype="<i4").tobytes()).digest()


def prompt_block_hashes(tokens, block_size: int) -> list:
    """Chained hashes of the full blocks of a prompt (a partial last block has none)."""
    out, parent = [], None
    for j in range(len(tokens) // block_size):
        parent = block_hash(parent, tokens[j * block_size:(j + 1) * block_size])
        out.append(parent)
    return out


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
        self.by_hash = {}          # prefix caching: hash -> block
        self.hash_of = {}          # block -> hash

    def allocate(self, n: int) -> list:
        if n < 0:
            raise ValueError("negative count")
        if len(self.free_blocks) < n:
            raise OutOfBlocks(f"Need {n} blocks, only {len(self.free_blocks)} available")
        taken = self.free_blocks[:n]
        self.free_blocks = self.free_blocks[n:]
        for b in taken:
            self.refcount[b] = 1
            self._drop_hash(b)     # new content: a cached hash no longer holds
        return taken

    def _drop_hash(self, b):
        h = self.hash_of.pop(b, None)
        if h is not None:
            del self.by_hash[h]

    def acquire_prefix(self, hashes):
        """Blocks for a prompt's full-block hashes, in order ([P4] Prefix
        Caching). A hash naming a cached block takes a reference to it (a
        cached block with no references left is taken back out of the free
        list); every other hash gets the head of the free list, registered
        under the hash. Cached blocks are taken before any fresh one, so a
        fresh allocation never evicts a block this request reuses. A block
        keeps its hash after it is freed and loses it when handed out again.
        Returns (ids, hits); OutOfBlocks leaves everything unchanged."""
        hashes = [bytes(h) for h in hashes]
        new_hashes = {h for h in hashes if h not in self.by_hash}
        revived = {self.by_hash[h] for h in hashes
                   if h in self.by_hash and self.refcount[self.by_hash[h]] == 0}
        if len(new_hashes) > len(self.free_blocks) - len(revived):
            raise OutOfBlocks(f"Need {len(new_hashes)} new blocks")
        ids, hits = [None] * len(hashes), 0
        for i, h in enumerate(hashes):
            if h in self.by_hash:
                b = self.by_hash[h]
                if self.refcount[b] == 0:
                    self.free_blocks.remove(b)
                self.refcount[b] += 1
                ids[i] = b
                hits += 1
        for i, h in enumerate(hashes):
            if ids[i] is not None:
                continue
            if h in self.by_hash:          # an earlier block of this request
                b = self.by_hash[h]
                self.refcount[b] += 1
                hits += 1
            else:
                (b,) = self.allocate(1)
                self.by_hash[h] = b
                self.hash_of[b] = h
            ids[i] = b
        return ids, hits

    def register_hash(self, block_id: int, h) -> None:
        """Give an allocated block (that just became full) its content hash;
        nothing happens if the hash names a block already."""
        b, h = int(block_id), bytes(h)
        if not (0 <= b < self.num_blocks) or self.refcount[b] == 0:
            raise ValueError("register_hash of a free or unknown block")
        if h in self.by_hash:
            return
        self._drop_hash(b)
        self.by_hash[h] = b
        self.hash_of[b] = h

    def lookup(self, h) -> int:
        return self.by_hash.get(bytes(h), -1)

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
