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


def _one_row_append(lib, row, dtype=torch.float32, n_kv=1, offset=0):
    """Quantise one token (one kv head unless n_kv > 1) into slot `offset` of a 1-block cache."""
    d = row.shape[-1]
    k = row.reshape(1, n_kv, d).to(dtype)
    v = (-row).reshape(1, n_kv, d).to(dtype)
    k8 = torch.zeros((1, n_kv, 16, d), dtype=torch.int8)
    v8 = torch.zeros((1, n_kv, d, 16), dtype=torch.int8)
    ks = torch.full((1, n_kv, 16), float("nan"))
    vs = torch.full((1, n_kv, 16), float("nan"))
    oracle.kv_append_int8(k, v, torch.tensor([offset]), k8, v8, ks, vs, lib=lib)
    return k8, v8, ks, vs


def pin_hand_worked_codes(lib):
    # amax 127 -> scale exactly 1.0: codes are rint(x).
    row = torch.tensor([127.0, -127.0, 3.0, 0.0, 64.4, -0.6, 12.5, 13.5])
    k8, _, ks, _ = _one_row_append(lib, row)
    assert float(ks[0, 0, 0]) == 1.0
    assert k8[0, 0, 0].tolist() == [127, -127, 3, 0, 64, -1, 12, 14]     # 12.5 -> 12, 13.5 -> 14 (half to even)
    # amax 254 -> scale 2.0: 1 / 2 = 0.5 is a tie -> 0; -100 / 2 = -50.
    row = torch.tensor([254.0, 1.0, -100.0, 3.0, 5.0, -5.0, 0.0, 253.0])
    k8, v8, ks, vs = _one_row_append(lib, row)
    assert float(ks[0, 0, 0]) == 2.0 and float(vs[0, 0, 0]) == 2.0
    assert k8[0, 0, 0].tolist() == [127, 0, -50, 2, 2, -2, 0, 126]      # 1.5 -> 2, 2.5 -> 2, 126.5 -> 126
    # An all-zero row has scale 0 and codes 0.
    k8, _, ks, _ = _one_row_append(lib, torch.zeros(8))
    assert float(ks[0, 0, 0]) == 0.0 and k8[0, 0, 0].abs().sum() == 0


def pin_rounding_bound(lib):
    g = torch.Generator().manual_seed(3)
    for dtype in (torch.bfloat16, torch.float16, torch.float32):
        rows = (torch.randn((64, 2, 128), generator=g) * torch.rand((64, 2, 1), generator=g) * 8).to(dtype)
        k8 = torch.zeros((4, 2, 16, 128), dtype=torch.int8)
        v8 = torch.zeros((4, 2, 128, 16), dtype=torch.int8)
        ks = torch.full((4, 2, 16), float("nan"))
        vs = torch.full((4, 2, 16), float("nan"))
        oracle.kv_append_int8(rows, rows, torch.arange(64), k8, v8, ks, vs, lib=lib)
        x = rows.double().numpy()                                  # [token, head, d]
        codes = k8.reshape(4, 2, 16, 128).permute(0, 2, 1, 3).reshape(64, 2, 128).double().numpy()
        sc = ks.permute(0, 2, 1).reshape(64, 2, 1).double().numpy()
        amax = np.abs(x).max(axis=2, keepdims=True)
        assert np.all(np.abs(codes) <= 127)
        assert np.all(np.abs(sc - amax / 127) <= amax / 127 * 2.0 ** -23)   # binary32 division
        assert np.all(np.abs(x - sc * codes) <= sc * (0.5 + 2.0 ** -16))
        # The largest element of every row is coded +-127.
        assert np.all(np.abs(np.take_along_axis(codes, np.abs(x).argmax(axis=2)[..., None], 2)) == 127)


def pin_transposed_v_positions(lib):
    # Token at block offset j lands at byte 4 * ((j % 8) / 2) + 2 * (j / 8) + (j % 2) of every V row.
    for j, pos in ((0, 0), (1, 1), (2, 4), (7, 13), (8, 2), (9, 3), (4, 8), (15, 15), (14, 14), (10, 6)):
        row = torch.arange(1, 9, dtype=torch.float32) * 10.0     # amax 80: codes rint(x * 127 / 80)
        k8, v8, ks, vs = _one_row_append(lib, row, offset=j)
        expect = torch.round(-row / float(vs[0, 0, j])).to(torch.int8)
        assert torch.equal(v8[0, 0, :, pos], expect), (j, pos)
        others = [p for p in range(16) if p != pos]
        assert v8[0, 0, :, others].abs().sum() == 0, (j, pos)
        assert torch.equal(k8[0, 0, j], -expect)


def _dequant_gather(w, k8, v8, ks, vs, b):
    bs, n_kv, d = w.block_size, w.n_kv_heads, w.head_dim
    pos = [4 * ((j % 8) // 2) + 2 * (j // 8) + (j % 2) for j in range(16)]
    n = int(w.context_lens[b])
    K = torch.empty((n_kv, n, d), dtype=torch.float64)
    V = torch.empty((n_kv, n, d), dtype=torch.float64)
    for j in range(n):
        blk, off = int(w.block_tables[b, j // bs]), j % bs
        K[:, j] = ks[blk, :, off, None].double() * k8[blk, :, off].double()
        V[:, j] = vs[blk, :, off, None].double() * v8[blk, :, :, pos[off]].double()
    return K, V


def pin_decode_equals_sdpa_on_dequantised(lib):
    w = build_workload("i8_sdpa", [1, 16, 17, 70, 33], 8, 2, 128, torch.bfloat16, seed=31)
    out, k8, v8, ks, vs = oracle.workload_decode_int8(w, lib=lib)
    G = w.n_q_heads // w.n_kv_heads
    for b in range(w.batch):
        K, V = _dequant_gather(w, k8, v8, ks, vs, b)
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


PINS = [pin_hand_worked_codes, pin_rounding_bound, pin_transposed_v_positions,
        pin_decode_equals_sdpa_on_dequantised, pin_placement_and_gqa, pin_close_to_unquantised]
