"""Seeded workload generators and the size arithmetic the pages print."""

import json
import math
from pathlib import Path

import torch

import workloads as W
from paged_kv_cache_386_b200 import layout

GOLDEN = Path(__file__).resolve().parent / "golden"


def test_kv_bytes_per_token_table():
    g = json.loads((GOLDEN / "kv_size_per_token.json").read_text())
    for row in g["rows"]:
        got = layout.kv_bytes_per_token(row["n_layers"], row["n_kv_heads"], row["head_dim"], row["elem_bytes"])
        assert got == row["bytes"], row["model"]
    assert layout.kv_bytes_per_token(80, 8, 128, 2) == g["worked_example_bytes"]
    assert 4096 * g["worked_example_bytes"] == g["llama3_70b_4k_context_gib"] * 2 ** 30
    assert 8192 * g["worked_example_bytes"] == g["llama3_70b_8k_context_gib"] * 2 ** 30


def test_best_of_8_block_counts():
    g = json.loads((GOLDEN / "best_of_8.json").read_text())
    gen = (g["private_token_blocks"] // g["samples"]) - g["prompt_tokens"]
    assert g["prompt_tokens"] + g["samples"] * gen == g["shared_token_blocks"]
    shared = W.best_of_n(prompts=1, n=8, prompt_len=2000, gen_len=gen, head_dim=64, n_q=8, n_kv=1,
                         pool_slack=0.0)
    private = W.build_workload("private", [2000 + gen] * 8, 8, 1, 64, torch.bfloat16, seed=0, pool_slack=0.0)
    assert shared.distinct_blocks == g["shared_blocks_16"]
    assert private.distinct_blocks == g["private_blocks_16"]
    tr = layout.decode_traffic(shared.block_tables, shared.context_lens, 8, 1, 64, 2)
    assert tr["unique_blocks"] == g["shared_blocks_16"] and tr["logical_blocks"] == g["private_blocks_16"]


def test_block_tables_are_consistent():
    w = W.uniform_gqa(batch=16, len_hi=600)
    used = []
    for b, n in enumerate(w.lens()):
        nb = layout.blocks_for(n)
        row = w.block_tables[b]
        assert (row[:nb] >= 0).all() and (row[nb:] == -1).all()
        used += row[:nb].tolist()
    assert len(set(used)) == len(used) == w.distinct_blocks   # private blocks, no reuse
    assert w.num_blocks == math.ceil(1.1 * w.distinct_blocks)
    # slot of the appended token = its logical position in its block
    for b, n in enumerate(w.lens()):
        s = int(w.slot_mapping[b])
        assert s // 16 == int(w.block_tables[b, (n - 1) // 16]) and s % 16 == (n - 1) % 16


def test_holes_hold_the_fill_value():
    w = W.uniform_gqa(batch=4, len_hi=300, head_dim=64)
    valid = torch.zeros(w.num_blocks, 16, dtype=torch.bool)
    for b, n in enumerate(w.lens()):
        for t in range(n - 1):   # the appended token's slot stays a hole
            valid[int(w.block_tables[b, t // 16]), t % 16] = True
    holes = (~valid).view(w.num_blocks, 1, 16, 1).expand_as(w.k_cache)
    assert torch.isnan(w.k_cache[holes].float()).all()
    assert not torch.isnan(w.k_cache[~holes].float()).any()


def test_length_distributions():
    a = W.uniform_gqa()
    assert min(a.lens()) >= 128 and max(a.lens()) <= 4096
    m = W.lognormal_mha()
    lens = sorted(m.lens())
    assert lens[0] >= 1 and lens[-1] <= 2048
    assert 200 <= lens[len(lens) // 2] <= 450    # median near 300
    s = W.shared_prefix(n_seqs=32, head_dim=64, n_q=8, n_kv=1)
    assert all(2048 + 16 <= n <= 2048 + 512 for n in s.lens())
    assert (s.block_tables[:, :128] == s.block_tables[0, :128]).all()   # one shared prefix


def test_long_context_pool_and_sinks():
    w = W.long_context(batch=2, ctx=4096, n_q=8, n_kv=2, head_dim=64)
    assert w.num_blocks == 2 * 256 == w.distinct_blocks
    ref = W.long_context(batch=2, ctx=4096, n_q=8, n_kv=2, head_dim=64, sink_scale=1.0)
    for b in range(2):
        p = int(w.block_tables[b, 0])
        assert torch.equal(w.k_cache[p, :, :4].float(), 4 * ref.k_cache[p, :, :4].float())
        assert torch.equal(w.k_cache[p, :, 4:].float(), ref.k_cache[p, :, 4:].float())


def test_generation_is_deterministic():
    a = W.uniform_gqa(batch=8, len_hi=500, head_dim=64, seed=3)
    b = W.uniform_gqa(batch=8, len_hi=500, head_dim=64, seed=3)
    for x, y in [(a.q, b.q), (a.block_tables, b.block_tables), (a.slot_mapping, b.slot_mapping)]:
        assert torch.equal(x, y)
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))


def test_identity_placement_is_consecutive_with_the_same_traffic():
    # bench.py --placement identity: the same sequences with each one's blocks
    # consecutive in the pool, sequences back to back; the bytes a decode must
    # read do not change.
    a = W.uniform_gqa(batch=6, seed=3)
    b = W.uniform_gqa(batch=6, seed=3, placement="identity")
    assert a.lens() == b.lens()
    assert torch.equal(a.q, b.q) and torch.equal(a.k_new, b.k_new)
    nxt = 0
    for s in range(b.batch):
        nb = layout.blocks_for(b.lens()[s])
        assert b.block_tables[s, :nb].tolist() == list(range(nxt, nxt + nb))
        nxt += nb
    args = (a.n_q_heads, a.n_kv_heads, a.head_dim, a.k_cache.element_size())
    assert (layout.decode_traffic(a.block_tables, a.context_lens, *args)
            == layout.decode_traffic(b.block_tables, b.context_lens, *args))
