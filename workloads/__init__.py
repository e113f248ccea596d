"""Seeded synthetic paged-decode workloads.

This module is shared by the CPU oracle tests, the GPU parity tests and
``bench.py``.  It draws the random numbers and lays out the paged cache:
context lengths, physical block placement, block tables, the slot of the
token appended this step, and the K/V/Q values.  It performs none of the
method's arithmetic: it never writes the appended token into the cache and
never computes attention.

Cache layout (shared by both sides of every parity check):

* ``k_cache``, ``v_cache``: ``[num_blocks, n_kv_heads, block_size, head_dim]``,
  row-major.  A physical block holds ``block_size`` consecutive tokens of
  one sequence (or of a shared prefix) for every kv head.
* ``block_tables``: ``int32 [batch, max_blocks_per_seq]``; entry ``j`` of row
  ``b`` is the physical block holding logical tokens ``16j .. 16j+15`` of
  sequence ``b`` (block table, "Transformer anatomy" ch. 15 §15.5; "LLM
  Primer VI" ch. 8 §8.1).  Unused entries hold -1.
* ``context_lens``: ``int32 [batch]``; counts the token appended this step.
* ``slot_mapping``: ``int64 [batch]``; ``block * block_size + offset`` of
  that token.

Slots that hold no token (the tail of the last block of a sequence, the
appended token's own slot before the append, free blocks) are filled with
``fill`` (NaN by default) so that a kernel that reads them into its result
is caught.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BLOCK_SIZE = 16

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
DTYPE_NAMES = {v: k for k, v in DTYPES.items()}


@dataclass
class DecodeWorkload:
    name: str
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    slot_mapping: torch.Tensor
    scale: float
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    block_size: int
    distinct_blocks: int
    appended: bool
    meta: dict = field(default_factory=dict)
    q_len: int = 1  # new tokens (queries) per sequence; q is [B, q_len, n_q, d] when > 1

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def num_blocks(self) -> int:
        return self.k_cache.shape[0]

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_tables.shape[1]

    @property
    def dtype(self) -> torch.dtype:
        return self.q.dtype

    @property
    def dtype_name(self) -> str:
        return DTYPE_NAMES[self.q.dtype]

    def lens(self) -> list[int]:
        return [int(x) for x in self.context_lens.tolist()]


def _blocks_for(n_tokens: int, block_size: int) -> int:
    return (n_tokens + block_size - 1) // block_size


def build_workload(
    name: str,
    lens: list[int],
    n_q_heads: int,
    n_kv_heads: int,
    head_dim: int,
    dtype: torch.dtype,
    seed: int,
    *,
    groups: list[tuple[list[int], int]] | None = None,
    pool_blocks: int | None = None,
    pool_slack: float = 0.10,
    placement: str = "shuffle",
    append: bool = True,
    fill: float = float("nan"),
    sink_tokens: int = 0,
    sink_scale: float = 1.0,
    scale: float | None = None,
    block_size: int = BLOCK_SIZE,
    max_blocks_per_seq: int | None = None,
    q_len: int = 1,
) -> DecodeWorkload:
    """Lay out ``len(lens)`` sequences in a shuffled pool of physical blocks.

    ``groups`` lists ``(member sequences, shared prefix tokens)``; the members
    of a group point their first ``prefix // block_size`` table entries at the
    same physical blocks (the refcounted sharing of "Transformer anatomy"
    ch. 15 §15.6 and "LLM Primer VI" ch. 8 §8.1).  ``prefix`` must be a
    multiple of ``block_size`` and shorter than every member's context, so
    that the appended token lands in a private block.

    ``q_len`` > 1 makes the last ``q_len`` tokens of every context new (their
    slots start at the fill value and ``k_new``/``v_new`` hold them, sequence
    major), with ``q`` of shape ``[B, q_len, n_q, d]``: several queries per
    sequence, as for verifying a draft or a prefill chunk.
    """
    assert q_len >= 1 and (q_len == 1 or (append and not sink_tokens))
    B = len(lens)
    g_struct = torch.Generator().manual_seed(seed)
    g_data = torch.Generator().manual_seed(seed + 7919)

    # Logical block -> distinct block id.  Shared prefix blocks first.
    seq_blocks: list[list[int]] = [[] for _ in range(B)]
    n_distinct = 0
    shared_of = [0] * B
    for members, prefix in groups or []:
        assert prefix % block_size == 0
        nshared = prefix // block_size
        ids = list(range(n_distinct, n_distinct + nshared))
        n_distinct += nshared
        for b in members:
            assert lens[b] > prefix, "appended token must land in a private block"
            seq_blocks[b] = list(ids)
            shared_of[b] = nshared
    for b in range(B):
        nb = _blocks_for(lens[b], block_size)
        extra = nb - len(seq_blocks[b])
        seq_blocks[b] += list(range(n_distinct, n_distinct + extra))
        n_distinct += extra

    if pool_blocks is None:
        pool_blocks = max(1, math.ceil((1.0 + pool_slack) * n_distinct))
    assert pool_blocks >= n_distinct
    if placement == "shuffle":
        phys_of = torch.randperm(pool_blocks, generator=g_struct)[:n_distinct]
    elif placement == "identity":
        phys_of = torch.arange(n_distinct)
    else:
        raise ValueError(placement)

    width = max(len(s) for s in seq_blocks) if B else 0
    if max_blocks_per_seq is not None:
        assert max_blocks_per_seq >= width
        width = max_blocks_per_seq
    width = max(width, 1)
    block_tables = torch.full((B, width), -1, dtype=torch.int32)
    for b in range(B):
        if seq_blocks[b]:
            block_tables[b, : len(seq_blocks[b])] = phys_of[torch.tensor(seq_blocks[b])].to(torch.int32)

    # How many leading slots of each physical block hold a token already
    # in the cache (the appended token's slot stays at the fill value).
    valid = torch.zeros(pool_blocks, dtype=torch.int64)
    for b in range(B):
        have = lens[b] - q_len if append else lens[b]
        for j, dblk in enumerate(seq_blocks[b]):
            n = min(block_size, have - j * block_size)
            if n <= 0:
                break
            p = int(phys_of[dblk])
            if n > valid[p]:
                valid[p] = n

    shape = (pool_blocks, n_kv_heads, block_size, head_dim)
    k_cache = _randn(shape, dtype, g_data)
    v_cache = _randn(shape, dtype, g_data)
    free = torch.nonzero(valid == 0).flatten()
    k_cache.index_fill_(0, free, fill)
    v_cache.index_fill_(0, free, fill)
    for p in torch.nonzero((valid > 0) & (valid < block_size)).flatten().tolist():
        n = int(valid[p])
        k_cache[p, :, n:, :] = fill
        v_cache[p, :, n:, :] = fill

    if sink_tokens:
        assert sink_tokens <= block_size
        for b in range(B):
            if lens[b] > 0:
                p = int(block_tables[b, 0])
                n = min(sink_tokens, lens[b] - (1 if append else 0))
                k_cache[p, :, :n, :] *= sink_scale

    q = _randn((B, n_q_heads, head_dim) if q_len == 1 else (B, q_len, n_q_heads, head_dim), dtype, g_data)
    k_new = _randn((B * q_len, n_kv_heads, head_dim), dtype, g_data)
    v_new = _randn((B * q_len, n_kv_heads, head_dim), dtype, g_data)
    if append and sink_tokens:
        for b in range(B):
            if lens[b] - 1 < sink_tokens:
                k_new[b] *= sink_scale

    slot = torch.full((B * q_len,), -1, dtype=torch.int64)
    if append:
        for b in range(B):
            for i in range(q_len):
                t = lens[b] - q_len + i
                if t >= 0:
                    slot[b * q_len + i] = int(block_tables[b, t // block_size]) * block_size + t % block_size

    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return DecodeWorkload(
        name=name, q=q, k_cache=k_cache, v_cache=v_cache, block_tables=block_tables,
        context_lens=torch.tensor(lens, dtype=torch.int32), k_new=k_new, v_new=v_new,
        slot_mapping=slot, scale=scale, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads,
        head_dim=head_dim, block_size=block_size, distinct_blocks=n_distinct, appended=append,
        meta={"seed": seed, "placement": placement, "pool_blocks": pool_blocks,
              "shared_blocks": shared_of, "groups": groups or []},
        q_len=q_len,
    )


def _randn(shape, dtype, gen, chunk_elems: int = 1 << 26) -> torch.Tensor:
    """N(0,1) drawn in float32 and rounded to ``dtype`` (chunked to bound memory)."""
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=gen, dtype=torch.float32).to(dtype)
    return out


@dataclass
class CascadeView:
    """The same workload split into shared prefixes and private suffixes."""
    prefix_block_tables: torch.Tensor  # int32 [n_groups, max_prefix_blocks]
    prefix_lens: torch.Tensor          # int32 [n_groups]
    seq_group: torch.Tensor            # int32 [batch], -1 = no group
    block_tables: torch.Tensor         # int32 [batch, max suffix blocks]
    context_lens: torch.Tensor         # int32 [batch] suffix tokens


def cascade_view(w: DecodeWorkload) -> CascadeView:
    """Table bookkeeping only: the shared prefix blocks of each group (from
    ``w.meta['groups']``) and, per sequence, the remaining private blocks."""
    groups = w.meta.get("groups", [])
    bs = w.block_size
    n_groups = len(groups)
    max_pb = max([pre // bs for _, pre in groups] + [1])
    ptab = torch.full((max(n_groups, 1), max_pb), -1, dtype=torch.int32)
    plen = torch.zeros(max(n_groups, 1), dtype=torch.int32)
    seq_group = torch.full((w.batch,), -1, dtype=torch.int32)
    for gi, (members, pre) in enumerate(groups):
        nb = pre // bs
        ptab[gi, :nb] = w.block_tables[members[0], :nb]
        plen[gi] = pre
        for b in members:
            seq_group[b] = gi
    skip = [int(plen[int(seq_group[b])]) // bs if seq_group[b] >= 0 else 0 for b in range(w.batch)]
    lens = [n - s * bs for n, s in zip(w.lens(), skip)]
    width = max(1, max((w.max_blocks_per_seq - s) for s in skip))
    tab = torch.full((w.batch, width), -1, dtype=torch.int32)
    for b in range(w.batch):
        row = w.block_tables[b, skip[b]:]
        tab[b, : row.numel()] = row
    return CascadeView(ptab[:n_groups] if n_groups else ptab[:0], plen[:n_groups], seq_group, tab,
                       torch.tensor(lens, dtype=torch.int32))


def cached_token_rows(w: DecodeWorkload):
    """Every slot that holds a token before this step's append, once each
    (shared blocks are listed once): ``(k_rows, v_rows, slots)`` with rows
    ``[n, n_kv, d]`` copied from the caches and int64 slots.  Used to fill a
    cache of another format with the same tokens."""
    bs = w.block_size
    slots = set()
    for b, n in enumerate(w.lens()):
        held = n - w.q_len if w.appended else n
        for j in range(held):
            slots.add(int(w.block_tables[b, j // bs]) * bs + j % bs)
    sl = torch.tensor(sorted(slots), dtype=torch.int64)
    blk, off = sl // bs, sl % bs
    k_rows = w.k_cache[blk, :, off, :].contiguous()
    v_rows = w.v_cache[blk, :, off, :].contiguous()
    return k_rows, v_rows, sl


def int8_cache_buffers(w: DecodeWorkload):
    """An empty INT8 cache for the pool of ``w``: uint8 records
    ``[blocks, n_kv, 32 * d + 128]`` with zero codes and NaN scales (the last
    128 bytes of each record), so that a read of a slot that holds no token
    poisons the result."""
    nb, nkv, bs, d = w.k_cache.shape
    cache = torch.zeros((nb, nkv, 32 * d + 128), dtype=torch.uint8)
    cache[:, :, 32 * d:].view(torch.float32).fill_(float("nan"))
    return cache


# ---------------------------------------------------------------------------
# The five workload shapes (Llama-class, block size 16).
# ---------------------------------------------------------------------------

def tiny_mha(seed: int = 0, **kw) -> DecodeWorkload:
    """4 sequences of context {1, 7, 16, 33}, 4 q = 4 kv heads, d=64, fp32, pool of 16."""
    return build_workload("tiny_mha_f32", [1, 7, 16, 33], 4, 4, 64, torch.float32, seed,
                          pool_blocks=16, **kw)


def uniform_gqa(batch: int = 64, n_q: int = 32, n_kv: int = 8, head_dim: int = 128,
                len_lo: int = 128, len_hi: int = 4096, dtype=torch.bfloat16, seed: int = 0,
                **kw) -> DecodeWorkload:
    """Llama-3-8B-shaped layer: GQA 4:1, context lengths uniform in [len_lo, len_hi]."""
    g = torch.Generator().manual_seed(seed + 101)
    lens = torch.randint(len_lo, len_hi + 1, (batch,), generator=g).tolist()
    return build_workload(f"llama3_8b_gqa_b{batch}", lens, n_q, n_kv, head_dim, dtype, seed, **kw)


def lognormal_mha(batch: int = 256, n_heads: int = 32, head_dim: int = 128, median: float = 300.0,
                  sigma: float = 1.0, clip: tuple[int, int] = (1, 2048), dtype=torch.float16,
                  seed: int = 0, **kw) -> DecodeWorkload:
    """Llama-2-7B-shaped MHA step: lengths round(clip(lognormal(ln median, sigma)))."""
    g = torch.Generator().manual_seed(seed + 202)
    x = torch.exp(math.log(median) + sigma * torch.randn(batch, generator=g, dtype=torch.float64))
    lens = torch.round(torch.clamp(x, clip[0], clip[1])).to(torch.int64).tolist()
    return build_workload(f"llama2_7b_mha_b{batch}", lens, n_heads, n_heads, head_dim, dtype, seed, **kw)


def shared_prefix(n_seqs: int = 128, prefix: int = 2048, suffix: tuple[int, int] = (16, 512),
                  n_q: int = 64, n_kv: int = 8, head_dim: int = 128, dtype=torch.bfloat16,
                  seed: int = 0, **kw) -> DecodeWorkload:
    """Llama-3-70B-shaped layer: every sequence shares one ``prefix``-token prefix."""
    g = torch.Generator().manual_seed(seed + 303)
    suf = torch.randint(suffix[0], suffix[1] + 1, (n_seqs,), generator=g).tolist()
    lens = [prefix + s for s in suf]
    return build_workload(f"shared_prefix_70b_n{n_seqs}", lens, n_q, n_kv, head_dim, dtype, seed,
                          groups=[(list(range(n_seqs)), prefix)], **kw)


def best_of_n(prompts: int = 16, n: int = 8, prompt_len: int = 2000, gen_len: int = 100,
              n_q: int = 64, n_kv: int = 8, head_dim: int = 128, dtype=torch.bfloat16,
              seed: int = 0, **kw) -> DecodeWorkload:
    """``prompts`` groups of ``n`` samples; each group shares its prompt's blocks."""
    assert prompt_len % BLOCK_SIZE == 0
    lens = [prompt_len + gen_len] * (prompts * n)
    groups = [(list(range(p * n, (p + 1) * n)), prompt_len) for p in range(prompts)]
    return build_workload(f"best_of_{n}_p{prompts}", lens, n_q, n_kv, head_dim, dtype, seed,
                          groups=groups, **kw)


def long_context(batch: int = 4, ctx: int = 131072, n_q: int = 64, n_kv: int = 8,
                 head_dim: int = 128, dtype=torch.bfloat16, seed: int = 0, sinks: int = 4,
                 sink_scale: float = 4.0, **kw) -> DecodeWorkload:
    """Long-context split-KV case: pool sized exactly for ``batch * ctx`` tokens,
    keys at positions 0..3 of each sequence scaled by 4 ("attention sinks")."""
    nb = _blocks_for(ctx, BLOCK_SIZE)
    kw.setdefault("pool_blocks", batch * nb)
    return build_workload(f"long_ctx_b{batch}_{ctx}", [ctx] * batch, n_q, n_kv, head_dim, dtype, seed,
                          sink_tokens=sinks, sink_scale=sink_scale, **kw)


CONFIGS = {
    "tiny_mha_f32": tiny_mha,
    "llama3_8b_gqa": uniform_gqa,
    "llama2_7b_mha": lognormal_mha,
    "shared_prefix_70b": shared_prefix,
    "best_of_8": best_of_n,
    "long_ctx_128k": long_context,
}
