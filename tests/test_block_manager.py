"""The library's C++ block manager (pkv_bm_* behind the C ABI) against the
reference model, operation by operation, on seeded random operation
sequences; plus the chained block keys and argument checks.  Host code only:
no GPU is needed."""

import random

import pytest
import torch

import oracle.block_manager as model
import paged_kv_cache_386_b200 as pkv


def _same_state(lib: pkv.BlockManager, ref: model.RefBlockManager, width: int):
    ids = sorted(ref.tables)
    bt, cl = lib.tables(ids, width)
    for row, s in enumerate(ids):
        t = ref.tables[s]
        assert bt[row, :len(t)].tolist() == t and bool((bt[row, len(t):] == -1).all())
        assert int(cl[row]) == ref.lengths[s]
    assert lib.stats() == ref.stats()
    assert [lib.refcount(b) for b in range(ref.num_blocks)] == ref.refcount


def _call(fn, *args):
    """Run one side; map its failure to a comparable token."""
    try:
        return ("ok", fn(*args))
    except model.NoBlocks:
        return ("no_blocks", None)
    except ValueError:
        return ("invalid", None)
    except pkv.PagedKVError as e:
        return ({pkv.PKV_ERR_NO_BLOCKS: "no_blocks", pkv.PKV_ERR_INVALID_ARG: "invalid"}[e.status], None)


def _fuzz(seed: int, num_blocks: int, prefix_cache: bool, steps: int, bs: int = 16):
    rng = random.Random(seed)
    width = num_blocks + 1
    lib = pkv.BlockManager(num_blocks, bs, prefix_cache=prefix_cache)
    ref = model.RefBlockManager(num_blocks, bs, prefix_cache=prefix_cache)
    base = [rng.randrange(1000) for _ in range(400)]
    prompts = [base[:rng.randrange(0, 400)] for _ in range(5)] + \
              [[rng.randrange(1000) for _ in range(rng.randrange(0, 200))] for _ in range(3)]
    live, next_id = [], 0
    for _ in range(steps):
        op = rng.random()
        if op < 0.2 or not live:
            p = rng.choice(prompts)
            keys = model.chained_block_keys(p, bs)
            assert pkv.pkv_bm_hash_blocks(p, bs) == keys
            a = _call(lib.add_sequence, next_id, len(p), keys)
            b = _call(ref.add_sequence, next_id, len(p), keys)
            assert a == b
            if a[0] == "ok":
                live.append(next_id)
            next_id += 1
        elif op < 0.3:
            parent = rng.choice(live)
            assert _call(lib.fork, parent, next_id) == _call(ref.fork, parent, next_id)
            live.append(next_id)
            next_id += 1
        elif op < 0.8:
            seqs = rng.sample(live, rng.randint(1, len(live)))
            a = _call(lib.append, seqs)
            b = _call(ref.append, seqs)
            assert a[0] == b[0]
            if a[0] == "ok":
                slots, src, dst = a[1]
                rslots, rcopies = b[1]
                assert slots.tolist() == rslots
                assert list(zip(src.tolist(), dst.tolist())) == rcopies
        else:
            s = rng.choice(live)
            live.remove(s)
            assert _call(lib.free, s) == _call(ref.free, s)
        _same_state(lib, ref, width)
    lib.close()


@pytest.mark.parametrize("seed,num_blocks,prefix_cache", [
    (1, 40, False), (2, 40, True), (3, 200, True), (4, 12, True), (5, 600, False), (6, 90, True),
])
def test_matches_reference_model(seed, num_blocks, prefix_cache):
    _fuzz(seed, num_blocks, prefix_cache, steps=500)


def test_best_of_8_through_the_library():
    # LLM Primer VI ch. 8 §8.1: 8 samples of a 2000-token prompt, 100 tokens each.
    bm = pkv.BlockManager(2048)
    bm.add_sequence(0, 2000)
    for c in range(1, 8):
        bm.fork(0, c)
    for _ in range(100):
        bm.append(list(range(8)))
    st = bm.stats()
    assert st["used_blocks"] == 181 and st["tokens"] == 8 * 2100


def test_chained_keys_match_model():
    rng = random.Random(3)
    toks = [rng.randrange(-2**31, 2**31) for _ in range(16 * 9 + 3)]
    for seed in (0, 1, 2**64 - 1):
        assert pkv.pkv_bm_hash_blocks(toks, 16, seed) == model.chained_block_keys(toks, 16, seed)
    assert pkv.pkv_bm_hash_blocks([], 16) == []


def test_argument_errors_change_nothing():
    bm = pkv.BlockManager(8)
    bm.add_sequence(1, 20)
    before = bm.stats()
    for bad in (lambda: bm.add_sequence(1, 5),            # existing id
                lambda: bm.add_sequence(2, -1),
                lambda: bm.fork(9, 10),                   # unknown parent
                lambda: bm.fork(1, 1),                    # existing child
                lambda: bm.append([1, 1]),                # duplicate
                lambda: bm.append([1, 5]),                # unknown
                lambda: bm.free(5),
                lambda: bm.tables([1], 1),                # table wider than the row
                lambda: bm.refcount(8)):
        with pytest.raises(pkv.PagedKVError) as e:
            bad()
        assert e.value.status == pkv.PKV_ERR_INVALID_ARG
    with pytest.raises(pkv.PagedKVError) as e:
        bm.add_sequence(3, 16 * 7 + 1)                    # needs 8 blocks, 6 free
    assert e.value.status == pkv.PKV_ERR_NO_BLOCKS
    assert bm.stats() == before
    with pytest.raises(pkv.PagedKVError):
        pkv.BlockManager(0)


def test_slot_mapping_feeds_append_layout():
    bm = pkv.BlockManager(64)
    bm.add_sequence(7, 31)
    slots, src, dst = bm.append([7])
    bt, cl = bm.tables([7], 4)
    assert int(cl[0]) == 32 and src.numel() == 0
    assert int(slots[0]) == int(bt[0, 1]) * 16 + 15
