"""Pins of the block-manager reference model (oracle/block_manager.py).

Each pin takes the model's module so that the planted-mistake test can run
the same pins against a mutated copy.  The pins come from the pages' numbers
(best-of-8 block counts, the 32-token shared prefix), the hash's published
test vectors, hand-worked LRU and copy-on-write traces, and invariants that
any correct allocator keeps (conservation of blocks, refcount = number of
table references, no two sequences writing one block, internal waste only
in the last block)."""

from __future__ import annotations

import json
import random
from pathlib import Path

GOLDEN = Path(__file__).resolve().parent / "golden"


def pin_fnv_vectors(m):
    for v in json.loads((GOLDEN / "fnv1a64_vectors.json").read_text())["vectors"]:
        assert m.fnv1a64(v["input_ascii"].encode()) == int(v["fnv1a64_hex"], 16), v


def pin_chained_keys_prefix_property(m):
    # Equal prefixes give equal keys; a change in block j changes keys j.. only.
    rng = random.Random(5)
    a = [rng.randrange(1 << 31) for _ in range(16 * 5)]
    b = list(a)
    b[16 * 2 + 7] ^= 1
    ka, kb = m.chained_block_keys(a), m.chained_block_keys(b)
    assert len(ka) == 5 and ka[:2] == kb[:2] and all(x != y for x, y in zip(ka[2:], kb[2:]))
    assert m.chained_block_keys(a[:16 * 3 + 5]) == ka[:3]          # partial block has no key
    assert m.chained_block_keys(a, seed=1) != ka


def pin_best_of_8_counts(m):
    g = json.loads((GOLDEN / "best_of_8.json").read_text())
    bs, prompt, n = g["block_size"], g["prompt_tokens"], g["samples"]
    gen = (g["private_token_blocks"] // n) - prompt
    shared = m.RefBlockManager(4096, bs)
    shared.add_sequence(0, prompt)
    for c in range(1, n):
        shared.fork(0, c)
    for _ in range(gen):
        shared.append(list(range(n)))
    assert shared.stats()["used_blocks"] == g["shared_blocks_16"]
    private = m.RefBlockManager(4096, bs)
    for c in range(n):
        private.add_sequence(c, prompt)
    for _ in range(gen):
        private.append(list(range(n)))
    assert private.stats()["used_blocks"] == g["private_blocks_16"]
    assert private.stats()["tokens"] == g["private_token_blocks"]


def pin_shared_prefix_example(m):
    g = json.loads((GOLDEN / "prefix_cache_example.json").read_text())
    bs, shared, total = g["block_size"], g["shared_prompt_tokens"], g["prompt_tokens"]
    p1 = list(range(1000, 1000 + total))
    p2 = p1[:shared] + [7] * (total - shared)
    bm = m.RefBlockManager(64, bs, prefix_cache=True)
    assert bm.add_sequence(1, total, m.chained_block_keys(p1, bs)) == 0
    assert bm.add_sequence(2, total, m.chained_block_keys(p2, bs)) == shared
    t1, t2 = bm.tables[1], bm.tables[2]
    assert len(t1) == len(t2) == g["blocks_per_prompt"]
    assert t1[:g["shared_blocks"]] == t2[:g["shared_blocks"]] and t1[2] != t2[2]
    assert bm.stats()["used_blocks"] == g["blocks_for_both_prompts"]


def pin_only_leading_run_shared(m):
    # A prefix hit is a prefix: once one block's key misses, later blocks are
    # not shared even if their keys are cached (their K/V were computed after
    # different earlier tokens).  Keys here are given directly, unchained.
    bm = m.RefBlockManager(16, 16, prefix_cache=True)
    bm.add_sequence(1, 48, [101, 102, 103])
    assert bm.add_sequence(2, 48, [101, 999, 103]) == 16
    assert bm.tables[2][0] == bm.tables[1][0]
    assert bm.tables[2][2] != bm.tables[1][2]
    assert bm.stats()["used_blocks"] == 5


def pin_fifo_lowest_free_and_tables(m):
    # "Transformer anatomy" §15.5: blocks come from the free pool as needed
    # and return to it when the sequence ends.
    bm = m.RefBlockManager(8, 16)
    bm.add_sequence(1, 33)           # blocks 0, 1, 2
    bm.add_sequence(2, 16)           # block 3
    slots, copies = bm.append([2, 1])
    assert bm.tables[1] == [0, 1, 2] and bm.tables[2] == [3, 4]
    assert slots == [4 * 16 + 0, 2 * 16 + 1] and copies == []
    bm.free(1)
    assert bm.stats()["free_blocks"] == 6
    bm.add_sequence(3, 20)           # lowest free: 0, 1
    assert bm.tables[3] == [0, 1]


def pin_copy_on_write_trace(m):
    bm = m.RefBlockManager(16, 16)
    bm.add_sequence(1, 40)           # blocks 0, 1, 2; the last holds 8 tokens
    bm.fork(1, 2)
    bm.fork(1, 3)
    assert [bm.refcount[b] for b in (0, 1, 2)] == [3, 3, 3]
    slots, copies = bm.append([2, 1, 3])
    # The first two writers copy the shared last block; the last writer is
    # then its only owner and writes in place.
    assert copies == [(2, 3), (2, 4)]
    assert slots == [3 * 16 + 8, 4 * 16 + 8, 2 * 16 + 8]
    assert bm.tables[1] == [0, 1, 4] and bm.tables[2] == [0, 1, 3] and bm.tables[3] == [0, 1, 2]
    assert [bm.refcount[b] for b in range(5)] == [3, 3, 1, 1, 1]
    bm.free(2)
    assert bm.refcount[0] == 2 and bm.refcount[3] == 0


def pin_lru_eviction_trace(m):
    bs = 16
    a = list(range(32))
    ka = m.chained_block_keys(a, bs)
    bm = m.RefBlockManager(4, bs, prefix_cache=True)
    bm.add_sequence(1, 32, ka)       # blocks 0, 1, both cached
    bm.free(1)                       # released last block first: idle order 1, 0
    assert bm.stats()["cached_idle_blocks"] == 2 and bm.stats()["free_blocks"] == 2
    bm.add_sequence(2, 48)           # free 2, 3, then evicts block 1 (released first)
    assert bm.tables[2] == [2, 3, 1]
    assert bm.stats()["cached_blocks"] == 1
    bm.free(2)                       # 1, 2, 3 hold no key: back to the free pool
    assert bm.add_sequence(3, 32, ka) == 16       # only block 0 is still cached
    assert bm.tables[3] == [0, 1]                  # block 1 re-registered under the second key
    bm.free(3)
    assert bm.add_sequence(4, 32, ka) == 32
    assert bm.tables[4] == [0, 1]


def pin_out_of_blocks_changes_nothing(m):
    bm = m.RefBlockManager(3, 16)
    bm.add_sequence(1, 32)
    bm.add_sequence(2, 16)
    before = (dict(bm.stats()), {k: list(v) for k, v in bm.tables.items()})
    try:
        bm.append([1, 2])            # needs 2 new blocks, 0 free
        raise AssertionError("append should have failed")
    except m.NoBlocks:
        pass
    assert (bm.stats(), bm.tables) == before


def pin_random_invariants(m):
    rng = random.Random(11)
    bs = 16
    bm = m.RefBlockManager(96, bs, prefix_cache=True)
    prompts = [[rng.randrange(50) for _ in range(rng.randrange(0, 120))] for _ in range(6)]
    live, next_id = [], 0
    for _ in range(600):
        op = rng.random()
        try:
            if op < 0.25 or not live:
                p = rng.choice(prompts)
                bm.add_sequence(next_id, len(p), m.chained_block_keys(p, bs))
                live.append(next_id)
                next_id += 1
            elif op < 0.35:
                bm.fork(rng.choice(live), next_id)
                live.append(next_id)
                next_id += 1
            elif op < 0.85:
                seqs = rng.sample(live, rng.randint(1, len(live)))
                slots, copies = bm.append(seqs)
                blocks = [s // bs for s in slots]
                assert len(set(slots)) == len(slots)
                assert all(bm.refcount[b] == 1 for b in blocks), "a written block is shared"
                assert all(bm.refcount[src] >= 1 and bm.refcount[dst] == 1 for src, dst in copies)
            else:
                s = rng.choice(live)
                live.remove(s)
                bm.free(s)
        except m.NoBlocks:
            pass
        st = bm.stats()
        assert st["free_blocks"] + st["cached_idle_blocks"] + st["used_blocks"] == bm.num_blocks
        refs = [0] * bm.num_blocks
        for t in bm.tables.values():
            for b in t:
                refs[b] += 1
        assert refs == bm.refcount
        for s, t in bm.tables.items():
            assert len(t) == -(-bm.lengths[s] // bs), "waste beyond the last block"


PINS = [pin_fnv_vectors, pin_chained_keys_prefix_property, pin_best_of_8_counts, pin_shared_prefix_example, pin_only_leading_run_shared,
        pin_fifo_lowest_free_and_tables, pin_copy_on_write_trace, pin_lru_eviction_trace,
        pin_out_of_blocks_changes_nothing, pin_random_invariants]
