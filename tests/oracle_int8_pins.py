"""Pins of the oracle's INT8 KV cache (quantising append and decode over the
dequantised cache), against facts that do not come from the oracle itself:
  * hand-worked codes for rows whose scale is exact, including a tie that
    rounds half to even;
  * the closed-form rounding bound |x - scale * code| <= scale / 2 (plus the
    binary32 division's rounding) on random rows;
  * the documented byte positions of tokens in the transposed V rows,
    computed by hand for a few offsets;
  * the decode equals torch scaled_dot_product_attention in fp64 on the
    gathered dequantised keys and values;
  * invariants: placement of blocks, GQA = repeated MHA.
``tests/test_oracle_int8.py`` runs them and the planted-mistake check."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from workloads import build_workload


def _rec(d):
    return 32 * d + 128


def _k_at(rec, j, e, d):
    """K code of (block offset j, dim e) read by the documented rule."""
    chunks = d // 16
    pos = j * d + ((e // 16) ^ (j % min(chunks, 8))) * 16 + e % 16
    return int(rec[pos].view(torch.int8))


def _v_at(rec, j, e, d):
    vpos = 4 * ((j % 8) // 2) + 2 * (j // 8) + (j % 2)
    return int(rec[16 * d + e * 16 + vpos].view(torch.int8))


def _scales(rec, j, d):
    f = rec[32 * d:].view(torch.float32)
    return float(f[j]), float(f[16 + j])


def _one_row_append(lib, row, dtype=torch.float32, offset=0):
    """Quantise one token (K = row, V = -row) into slot `offset` of a 1-block, 1-head cache."""
    d = row.shape[-1]
    k = row.reshape(1, 1, d).to(dtype)
    v = (-row).reshape(1, 1, d).to(dtype)
    cache = torch.zeros((1, 1, _rec(d)), dtype=torch.uint8)
    cache[:, :, 32 * d:].view(torch.float32).fill_(float("nan"))
    oracle.kv_append_int8(k, v, torch.tensor([offset]), cache, lib=lib)
    return cache[0, 0]


def _codes(rec, j, d, which):
    get = _k_at if which == "k" else _v_at
    return [get(rec, j, e, d) for e in range(d)]


def pin_hand_worked_codes(lib):
    d = 64
    # amax 127 -> scale exactly 1.0: codes are rint(x).
    head = [127.0, -127.0, 3.0, 0.0, 64.4, -0.6, 12.5, 13.5]
    row = torch.tensor(head + [0.0] * (d - 8))
    rec = _one_row_append(lib, row)
    assert _scales(rec, 0, d) == (1.0, 1.0)
    assert _codes(rec, 0, d, "k")[:8] == [127, -127, 3, 0, 64, -1, 12, 14]     # 12.5 -> 12, 13.5 -> 14
    # amax 254 -> scale 2.0: 1 / 2 = 0.5 is a tie -> 0; -100 / 2 = -50.
    head = [254.0, 1.0, -100.0, 3.0, 5.0, -5.0, 0.0, 253.0]
    rec = _one_row_append(lib, torch.tensor(head + [0.0] * (d - 8)))
    assert _scales(rec, 0, d) == (2.0, 2.0)
    assert _codes(rec, 0, d, "k")[:8] == [127, 0, -50, 2, 2, -2, 0, 126]      # 1.5 -> 2, 2.5 -> 2, 126.5 -> 126
    assert _codes(rec, 0, d, "v")[:8] == [-127, 0, 50, -2, -2, 2, 0, -126]
    # An all-zero row has scale 0 and codes 0.
    rec = _one_row_append(lib, torch.zeros(d))
    assert _scales(rec, 0, d)[0] == 0.0 and not any(_codes(rec, 0, d, "k"))


def pin_rounding_bound(lib):
    g = torch.Generator().manual_seed(3)
    for dtype, d in ((torch.bfloat16, 128), (torch.float16, 64), (torch.float32, 128)):
        rows = (torch.randn((64, 2, d), generator=g) * torch.rand((64, 2, 1), generator=g) * 8).to(dtype)
        cache = torch.zeros((4, 2, _rec(d)), dtype=torch.uint8)
        oracle.kv_append_int8(rows, rows, torch.arange(64), cache, lib=lib)
        for i in range(0, 64, 7):
            for h in range(2):
                rec = cache[i // 16, h]
                x = rows[i, h].double()
                sk, sv = _scales(rec, i % 16, d)
                amax = x.abs().max().item()
                assert abs(sk - amax / 127) <= amax / 127 * 2.0 ** -23 and sk == sv
                for which in ("k", "v"):
                    c = torch.tensor(_codes(rec, i % 16, d, which), dtype=torch.float64)
                    assert c.abs().max().item() == 127 if amax > 0 else True
                    assert ((x - sk * c).abs() <= sk * (0.5 + 2.0 ** -16)).all()


def pin_record_positions(lib):
    # K code of dim e at block offset j: chunk (e / 16) ^ (j % 8) of row j
    # (d = 128); V code at byte 4 * ((j % 8) / 2) + 2 * (j / 8) + (j % 2) of
    # row e of the transposed part; scales at 32 d + 4 j and 32 d + 64 + 4 j.
    d = 128
    row = torch.zeros(d)
    row[37] = 5.0                         # dim 37: chunk 2, byte 5 of the chunk
    for j, kchunk, vbyte in ((0, 2, 0), (1, 3, 1), (3, 1, 5), (5, 7, 9), (9, 3, 3), (12, 6, 10), (15, 5, 15)):
        rec = _one_row_append(lib, row, offset=j)
        assert rec[j * d + kchunk * 16 + 5].view(torch.int8).item() == 127, (j, kchunk)
        assert rec[16 * d + 37 * 16 + vbyte].view(torch.int8).item() == -127, (j, vbyte)
        nz = torch.nonzero(rec[: 32 * d]).flatten().tolist()
        assert nz == [j * d + kchunk * 16 + 5, 16 * d + 37 * 16 + vbyte], (j, nz)
        assert rec[32 * d + 4 * j: 32 * d + 4 * j + 4].view(torch.float32).item() == \
            torch.tensor(5.0, dtype=torch.float32).div(127).item()


def _dequant_gather(w, cache, b):
    bs, n_kv, d = w.block_size, w.n_kv_heads, w.head_dim
    n = int(w.context_lens[b])
    K = torch.empty((n_kv, n, d), dtype=torch.float64)
    V = torch.empty((n_kv, n, d), dtype=torch.float64)
    for j in range(n):
        blk, off = int(w.block_tables[b, j // bs]), j % bs
        for h in range(n_kv):
            rec = cache[blk, h]
            sk, sv = _scales(rec, off, d)
            K[h, j] = sk * torch.tensor(_codes(rec, off, d, "k"), dtype=torch.float64)
            V[h, j] = sv * torch.tensor(_codes(rec, off, d, "v"), dtype=torch.float64)
    return K, V


def pin_decode_equals_sdpa_on_dequantised(lib):
    w = build_workload("i8_sdpa", [1, 16, 17, 70, 33], 8, 2, 128, torch.bfloat16, seed=31)
    out, cache = oracle.workload_decode_int8(w, lib=lib)
    G = w.n_q_heads // w.n_kv_heads
    for b in range(w.batch):
        K, V = _dequant_gather(w, cache, b)
        q = w.q[b].double().reshape(w.n_kv_heads, G, 1, w.head_dim)
        ref = torch.nn.functional.scaled_dot_product_attention(q, K[:, None], V[:, None], scale=w.scale)
        err = (out[b] - ref.reshape(w.n_q_heads, w.head_dim)).abs().max().item()
        assert err < 1e-12, (b, err)


def pin_placement_and_gqa(lib):
    w = build_workload("i8_perm", [40, 5, 64], 8, 2, 128, torch.float16, seed=32)
    a, *_ = oracle.workload_decode_int8(w, lib=lib)
    # Same tokens, other physical placement: identical bits.
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(1))
    m = build_workload("i8_perm", [40, 5, 64], 8, 2, 128, torch.float16, seed=32)
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(w.num_blocks)
    m.k_cache, m.v_cache = w.k_cache[inv].clone(), w.v_cache[inv].clone()
    m.block_tables = torch.where(w.block_tables >= 0, perm[w.block_tables.clamp(min=0).long()].int(),
                                 w.block_tables)
    m.slot_mapping = perm[w.slot_mapping // 16] * 16 + w.slot_mapping % 16
    b, *_ = oracle.workload_decode_int8(m, lib=lib)
    assert torch.equal(a, b)
    # GQA = MHA with the kv heads repeated.
    G = w.n_q_heads // w.n_kv_heads
    r = build_workload("i8_perm", [40, 5, 64], 8, 2, 128, torch.float16, seed=32)
    r.n_kv_heads = w.n_q_heads
    r.k_cache = w.k_cache.repeat_interleave(G, dim=1).contiguous()
    r.v_cache = w.v_cache.repeat_interleave(G, dim=1).contiguous()
    r.k_new = w.k_new.repeat_interleave(G, dim=1).contiguous()
    r.v_new = w.v_new.repeat_interleave(G, dim=1).contiguous()
    c, *_ = oracle.workload_decode_int8(r, lib=lib)
    assert torch.equal(a, c)


def pin_close_to_unquantised(lib):
    w = build_workload("i8_close", [300, 1000, 77], 32, 8, 128, torch.bfloat16, seed=33)
    q8, *_ = oracle.workload_decode_int8(w, lib=lib)
    ref, _, _ = oracle.workload_decode(w, lib=lib)
    rel = ((q8 - ref).norm() / ref.norm()).item()
    assert 1e-4 < rel < 2e-2, rel       # 8-bit codes: visible but small


PINS = [pin_hand_worked_codes, pin_rounding_bound, pin_record_positions,
        pin_decode_equals_sdpa_on_dequantised, pin_placement_and_gqa, pin_close_to_unquantised]
