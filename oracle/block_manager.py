"""Reference model of the paged KV block manager (test infrastructure only).

This is a plain, slow, dictionary-and-list restatement of the allocator that
hands out the block tables and slots the kernels read.  Only the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU leg use it; it shares no
code with the library's C++ manager.

What it follows:

* "Transformer anatomy" ch. 15 §15.5: a pool of fixed 16-token blocks, a
  per-sequence block table, a new token goes into the last block and a new
  block is taken from the free pool when that block is full, a finished
  sequence returns its blocks to the pool.
* "LLM Primer VI" ch. 8 §8.1: block tables of different sequences may point
  at one physical block, counted by a refcount (parallel sampling).  Writing
  into a shared block is read as copy-on-write: the writer moves to a fresh
  copy first.
* "Transformer anatomy" ch. 15 §15.6 and "LLM Primer VI" ch. 8 §8.3: prompt
  blocks are keyed by a hash, a new prompt whose leading keys are cached
  points its table at the cached blocks and skips their prefill, and cached
  blocks are evicted least recently used first.  A block's key is read as
  covering every token up to the block's end (a chain of hashes), because a
  block's K/V depend on the whole prefix before it.

Readings fixed so that two implementations can agree step by step: a new
block is the lowest-numbered free block; with none free, the cached block
released longest ago is evicted; freeing a sequence releases its blocks from
the last to the first; an append that cannot be served changes nothing.

The chained key uses FNV-1a 64 (Fowler, Noll, Vo: offset basis
14695981039346656037, prime 1099511628211, for each byte xor then multiply
modulo 2^64) over the 8 little-endian bytes of the previous key followed by
the block's tokens as 4-byte little-endian integers.
"""

from __future__ import annotations

import struct

FNV_OFFSET = 14695981039346656037
FNV_PRIME = 1099511628211
MASK64 = (1 << 64) - 1


class NoBlocks(Exception):
    """The pool cannot supply the blocks an operation needs."""


def fnv1a64(data: bytes, h: int = FNV_OFFSET) -> int:
    for byte in data:
        h ^= byte
        h = (h * FNV_PRIME) & MASK64
    return h


def chained_block_keys(tokens, block_size: int = 16, seed: int = 0) -> list[int]:
    keys, prev = [], seed & MASK64
    for i in range(len(tokens) // block_size):
        chunk = tokens[i * block_size:(i + 1) * block_size]
        data = struct.pack("<Q", prev) + b"".join(struct.pack("<I", int(t) & 0xFFFFFFFF) for t in chunk)
        prev = fnv1a64(data)
        keys.append(prev)
    return keys


class RefBlockManager:
    def __init__(self, num_blocks: int, block_size: int = 16, prefix_cache: bool = False):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.prefix_cache = prefix_cache
        self.refcount = [0] * num_blocks
        self.key_of_block: dict[int, int] = {}   # cached block -> its key
        self.block_of_key: dict[int, int] = {}   # key -> cached block
        self.idle: list[int] = []                # cached blocks with refcount 0, oldest release first
        self.tables: dict[int, list[int]] = {}   # sequence -> block table
        self.lengths: dict[int, int] = {}        # sequence -> tokens

    # -- pool ---------------------------------------------------------------
    def free_list(self) -> list[int]:
        return [b for b in range(self.num_blocks) if self.refcount[b] == 0 and b not in self.key_of_block]

    def available(self) -> int:
        return len(self.free_list()) + len(self.idle)

    def _take(self) -> int:
        free = self.free_list()
        if free:
            b = free[0]
        else:
            b = self.idle.pop(0)
            del self.block_of_key[self.key_of_block.pop(b)]
        self.refcount[b] = 1
        return b

    def _release(self, b: int) -> None:
        self.refcount[b] -= 1
        if self.refcount[b] == 0 and b in self.key_of_block:
            self.idle.append(b)

    # -- operations ---------------------------------------------------------
    def add_sequence(self, seq: int, n_tokens: int, keys=None) -> int:
        if seq in self.tables or n_tokens < 0:
            raise ValueError("bad sequence")
        bs = self.block_size
        n_blocks = -(-n_tokens // bs)
        n_full = n_tokens // bs
        hit_blocks = []
        if self.prefix_cache and keys is not None:
            for i in range(n_full):
                if keys[i] not in self.block_of_key:
                    break
                hit_blocks.append(self.block_of_key[keys[i]])
        leaving_idle = sum(1 for b in hit_blocks if self.refcount[b] == 0)
        if self.available() - leaving_idle < n_blocks - len(hit_blocks):
            raise NoBlocks()
        table = []
        for b in hit_blocks:
            if self.refcount[b] == 0:
                self.idle.remove(b)
            self.refcount[b] += 1
            table.append(b)
        for i in range(len(hit_blocks), n_blocks):
            b = self._take()
            table.append(b)
            if self.prefix_cache and keys is not None and i < n_full and keys[i] not in self.block_of_key:
                self.block_of_key[keys[i]] = b
                self.key_of_block[b] = keys[i]
        self.tables[seq] = table
        self.lengths[seq] = n_tokens
        return len(hit_blocks) * bs

    def fork(self, parent: int, child: int) -> None:
        if parent not in self.tables or child in self.tables:
            raise ValueError("bad fork")
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for b in self.tables[child]:
            self.refcount[b] += 1

    def append(self, seqs):
        if len(set(seqs)) != len(seqs) or any(s not in self.tables for s in seqs):
            raise ValueError("bad append")
        bs = self.block_size
        need = 0
        for s in seqs:
            if self.lengths[s] % bs == 0 or self.refcount[self.tables[s][-1]] > 1:
                need += 1
        if self.available() < need:
            raise NoBlocks()
        slots, copies = [], []
        for s in seqs:
            offset = self.lengths[s] % bs
            table = self.tables[s]
            if offset == 0:
                table.append(self._take())
            elif self.refcount[table[-1]] > 1:
                old = table[-1]
                new = self._take()
                self._release(old)
                table[-1] = new
                copies.append((old, new))
            slots.append(table[-1] * bs + offset)
            self.lengths[s] += 1
        return slots, copies

    def free(self, seq: int) -> None:
        table = self.tables.pop(seq)
        del self.lengths[seq]
        for b in reversed(table):
            self._release(b)

    def stats(self) -> dict:
        free = len(self.free_list())
        return {
            "num_blocks": self.num_blocks,
            "free_blocks": free,
            "cached_idle_blocks": len(self.idle),
            "used_blocks": self.num_blocks - free - len(self.idle),
            "cached_blocks": len(self.key_of_block),
            "sequences": len(self.tables),
            "tokens": sum(self.lengths.values()),
            "allocated_slots": sum(len(t) for t in self.tables.values()) * self.block_size,
        }
