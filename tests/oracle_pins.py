"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each ``pin_*`` function takes a loaded oracle library handle and raises
``AssertionError`` when the oracle disagrees with
  * the exact high-precision brute force (``oracle.brute``),
  * a library routine (torch ``scaled_dot_product_attention`` in fp64),
  * a closed form (context 1 returns V; equal keys or scale 0 return the mean
    of V), or
  * an invariant of the method (block placement, shared blocks, GQA = MHA
    with repeated kv heads).
``tests/test_oracle_pins.py`` runs them on the real oracle and
``tests/test_oracle_mutants.py`` checks that every planted mistake in the
oracle's C source fails at least one of them.
"""

from __future__ import annotations

import json
import math
from pathlib import Path

import numpy as np
import torch

import oracle
from oracle import brute
from workloads import build_workload, tiny_mha

GOLDEN = Path(__file__).resolve().parent / "golden"


def _run(lib, w, rows=None):
    out, _, _ = oracle.workload_decode(w, rows=rows, lib=lib)
    return out


def _lists(t):
    return t.double().tolist()


def _brute(w, kc, vc):
    return torch.tensor(brute.attention_rows(
        _lists(w.q), _lists(kc), _lists(vc), w.block_tables.tolist(), w.context_lens.tolist(),
        w.scale, w.n_q_heads, w.n_kv_heads, w.block_size), dtype=torch.float64)


def pin_brute_force_tiny(lib):
    """The tiny MHA fp32 case and small GQA bf16 / f16 cases against the
    50-digit decimal brute force (append included)."""
    cases = [
        tiny_mha(seed=0),
        build_workload("gqa_bf16", [3, 17, 32], 4, 2, 64, torch.bfloat16, seed=5, pool_blocks=9),
        build_workload("gqa_f16", [20, 1], 6, 2, 64, torch.float16, seed=6, pool_blocks=5),
    ]
    for w in cases:
        out, kc, vc = oracle.workload_decode(w, lib=lib)
        ref = _brute(w, kc, vc)
        err = (out - ref).abs().max().item()
        assert err < 1e-13, f"{w.name}: oracle vs brute force max err {err}"


def pin_context_one_returns_v(lib):
    """Context length 1: the only weight is exp(0)/exp(0) = 1, so the output
    is the appended V row exactly."""
    w = build_workload("ctx1", [1, 1, 1], 8, 2, 128, torch.bfloat16, seed=11)
    out = _run(lib, w)
    G = w.n_q_heads // w.n_kv_heads
    for b in range(w.batch):
        for h in range(w.n_q_heads):
            assert torch.equal(out[b, h], w.v_new[b, h // G].double()), (b, h)


def pin_equal_keys_mean_v(lib):
    """All keys of a sequence equal: uniform weights, the output is the mean
    of the V rows (numpy mean of the gathered rows)."""
    w = build_workload("eqk", [5, 40, 16], 4, 4, 64, torch.float32, seed=12, append=False)
    kc = w.k_cache
    key = torch.randn(64, generator=torch.Generator().manual_seed(3))
    for b, n in enumerate(w.lens()):
        for t in range(n):
            kc[int(w.block_tables[b, t // 16]), :, t % 16, :] = key
    out = _run(lib, w)
    for b, n in enumerate(w.lens()):
        for h in range(w.n_q_heads):
            rows = np.stack([w.v_cache[int(w.block_tables[b, t // 16]), h, t % 16].double().numpy()
                             for t in range(n)])
            assert np.allclose(out[b, h].numpy(), rows.mean(axis=0), rtol=0, atol=1e-14)


def pin_scale_zero_mean_v(lib):
    """scale = 0: every score is 0, the output is the mean of V."""
    w = build_workload("s0", [9, 33], 4, 2, 64, torch.float16, seed=13, append=False, scale=0.0)
    out = _run(lib, w)
    for b, n in enumerate(w.lens()):
        for h in range(w.n_q_heads):
            rows = np.stack([w.v_cache[int(w.block_tables[b, t // 16]), h // 2, t % 16].double().numpy()
                             for t in range(n)])
            assert np.allclose(out[b, h].numpy(), rows.mean(axis=0), rtol=0, atol=1e-14)


def pin_paged_equals_dense_sdpa(lib):
    """Gathered through the table, paged attention equals dense
    scaled-dot-product attention (torch SDPA in fp64, GQA by repeat of kv
    heads in contiguous groups)."""
    w = build_workload("dense", [1, 15, 16, 17, 70], 8, 2, 64, torch.bfloat16, seed=14, append=False)
    out = _run(lib, w)
    G = w.n_q_heads // w.n_kv_heads
    for b, n in enumerate(w.lens()):
        phys = [int(w.block_tables[b, t // 16]) for t in range(n)]
        off = [t % 16 for t in range(n)]
        K = torch.stack([w.k_cache[p, :, o, :] for p, o in zip(phys, off)], dim=1).double()  # [kv, n, d]
        V = torch.stack([w.v_cache[p, :, o, :] for p, o in zip(phys, off)], dim=1).double()
        K = K.repeat_interleave(G, dim=0)
        V = V.repeat_interleave(G, dim=0)
        qb = w.q[b].double().unsqueeze(1)  # [h, 1, d]
        ref = torch.nn.functional.scaled_dot_product_attention(qb, K, V, scale=w.scale).squeeze(1)
        err = (out[b] - ref).abs().max().item()
        assert err < 1e-12, f"seq {b}: {err}"


def pin_permutation_invariance(lib):
    """Moving physical blocks around (tables rewritten to match) changes no
    bit of the output."""
    w = build_workload("perm", [30, 64, 3, 100], 8, 4, 64, torch.bfloat16, seed=15)
    out = _run(lib, w)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(99))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(w.num_blocks)
    w2 = build_workload("perm", [30, 64, 3, 100], 8, 4, 64, torch.bfloat16, seed=15)
    w2.k_cache = w.k_cache[inv].clone()   # new block p holds old block inv[p]
    w2.v_cache = w.v_cache[inv].clone()
    bt = w.block_tables.clone()
    used = bt >= 0
    bt[used] = perm[bt[used].long()].to(torch.int32)
    w2.block_tables = bt
    s = w.slot_mapping.clone()
    s = perm[(s // 16)] * 16 + s % 16
    w2.slot_mapping = s
    out2 = _run(lib, w2)
    assert torch.equal(out, out2)


def pin_shared_equals_private(lib):
    """Sequences that share prefix blocks give the same bits as the same
    sequences with private copies of those blocks."""
    lens = [48 + 5, 48 + 20, 48 + 1]
    shared = build_workload("sh", lens, 4, 2, 64, torch.bfloat16, seed=16,
                            groups=[([0, 1, 2], 48)])
    out = _run(lib, shared)
    # Private copy: give each sequence its own copy of the 3 prefix blocks.
    pb = shared.block_tables[0, :3].tolist()
    extra = len(lens) * 3
    kc = torch.cat([shared.k_cache, torch.empty((extra,) + shared.k_cache.shape[1:], dtype=shared.k_cache.dtype)])
    vc = torch.cat([shared.v_cache, torch.empty((extra,) + shared.v_cache.shape[1:], dtype=shared.v_cache.dtype)])
    bt = shared.block_tables.clone()
    nxt = shared.num_blocks
    for b in range(len(lens)):
        for j, p in enumerate(pb):
            kc[nxt] = shared.k_cache[p]
            vc[nxt] = shared.v_cache[p]
            bt[b, j] = nxt
            nxt += 1
    shared.k_cache, shared.v_cache, shared.block_tables = kc, vc, bt
    out2 = _run(lib, shared)
    assert torch.equal(out, out2)


def pin_gqa_equals_repeated_mha(lib):
    """GQA with G = n_q / n_kv equals MHA whose kv head h is kv head h / G of
    the GQA cache (contiguous groups)."""
    w = build_workload("gqa", [25, 49], 8, 2, 64, torch.float16, seed=17)
    out = _run(lib, w)
    G = 4
    m = build_workload("gqa", [25, 49], 8, 2, 64, torch.float16, seed=17)
    m.k_cache = w.k_cache.repeat_interleave(G, dim=1).contiguous()
    m.v_cache = w.v_cache.repeat_interleave(G, dim=1).contiguous()
    m.k_new = w.k_new.repeat_interleave(G, dim=1).contiguous()
    m.v_new = w.v_new.repeat_interleave(G, dim=1).contiguous()
    m.n_kv_heads = 8
    out2 = _run(lib, m)
    assert torch.equal(out, out2)


def pin_block_table_example(lib):
    """The two block tables of the PagedAttention figure ([1, 4, 6] and
    [2, 7]; blocks 3, 5, 8 free): free blocks hold NaN and are never read;
    the result equals dense attention over the gathered tokens."""
    g = json.loads((GOLDEN / "block_table_example.json").read_text())
    tables = g["block_tables"]
    lens = [16 * (len(tables[0]) - 1) + 9, 16 * (len(tables[1]) - 1) + 16]  # ragged tail, full tail
    w = build_workload("fig", lens, 2, 2, 64, torch.float32, seed=18, pool_blocks=9,
                       placement="identity", append=False)
    gen = torch.Generator().manual_seed(19)
    kc = torch.full_like(w.k_cache, float("nan"))
    vc = torch.full_like(w.v_cache, float("nan"))
    for b, tab in enumerate(tables):
        for t in range(lens[b]):
            kc[tab[t // 16], :, t % 16, :] = torch.randn(2, 64, generator=gen)
            vc[tab[t // 16], :, t % 16, :] = torch.randn(2, 64, generator=gen)
    bt = torch.full((2, 3), -1, dtype=torch.int32)
    for b, tab in enumerate(tables):
        bt[b, : len(tab)] = torch.tensor(tab, dtype=torch.int32)
    w.k_cache, w.v_cache, w.block_tables = kc, vc, bt
    out = _run(lib, w)
    assert torch.isfinite(out).all()
    for b, tab in enumerate(tables):
        K = torch.stack([kc[tab[t // 16], :, t % 16, :] for t in range(lens[b])], dim=1).double()
        V = torch.stack([vc[tab[t // 16], :, t % 16, :] for t in range(lens[b])], dim=1).double()
        ref = torch.nn.functional.scaled_dot_product_attention(
            w.q[b].double().unsqueeze(1), K, V, scale=w.scale).squeeze(1)
        assert (out[b] - ref).abs().max().item() < 1e-12


def pin_append_roundtrip(lib):
    """After the append, slot s of every kv head holds the new K/V row bit for
    bit; every other slot keeps its canary bits; negative slots are skipped."""
    num_blocks, n_kv, bs, d = 6, 3, 16, 64
    for dtype in (torch.float32, torch.float16, torch.bfloat16):
        canary = torch.full((num_blocks, n_kv, bs, d), 0.0, dtype=dtype)
        canary.view(torch.int16 if dtype != torch.float32 else torch.int32).fill_(0x3A5C)
        kc, vc = canary.clone(), canary.clone()
        gen = torch.Generator().manual_seed(20)
        slots = torch.tensor([0, 17, -1, 95, 40, -7], dtype=torch.int64)
        k = torch.randn(len(slots), n_kv, d, generator=gen).to(dtype)
        v = torch.randn(len(slots), n_kv, d, generator=gen).to(dtype)
        oracle.kv_append(k, v, slots, kc, vc, bs, lib=lib)
        touched = torch.zeros(num_blocks, bs, dtype=torch.bool)
        for i, s in enumerate(slots.tolist()):
            if s < 0:
                continue
            assert torch.equal(kc[s // bs, :, s % bs], k[i]) and torch.equal(vc[s // bs, :, s % bs], v[i])
            touched[s // bs, s % bs] = True
        mask = (~touched).view(num_blocks, 1, bs, 1).expand_as(kc)
        assert torch.equal(kc[mask], canary[mask]) and torch.equal(vc[mask], canary[mask])


def pin_widening(lib):
    """The oracle's own f16/bf16 -> double conversions agree with numpy's
    float16 and torch's bfloat16 on all 65,536 bit patterns."""
    bits = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16)
    for dtype in (torch.float16, torch.bfloat16):
        t = bits.view(dtype).clone()
        got = oracle.widen(t, lib=lib)
        if dtype == torch.float16:
            ref = t.numpy().astype(np.float64)
        else:
            ref = t.double().numpy()
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(got), nan)
        assert np.array_equal(got[~nan], ref[~nan])


PINS = [pin_brute_force_tiny, pin_context_one_returns_v, pin_equal_keys_mean_v,
        pin_scale_zero_mean_v, pin_paged_equals_dense_sdpa, pin_permutation_invariance,
        pin_shared_equals_private, pin_gqa_equals_repeated_mha, pin_block_table_example,
        pin_append_roundtrip, pin_widening]
