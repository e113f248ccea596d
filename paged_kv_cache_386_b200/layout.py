"""Byte accounting of the paged KV cache (host side, no GPU).

* :func:`kv_bytes_per_token` is the per-token cache size of a whole model:
  layers x 2 (K and V) x kv heads x head dim x element bytes ("Transformer
  anatomy" ch. 15 §15.2, size-per-token formula and table).
* :func:`decode_traffic` counts the algorithmic HBM bytes of one
  ``paged_attention_decode`` call: the K and V tile of every distinct
  (physical block, kv head) pair that some sequence reads (a partial tail
  block counts whole, since it is loaded whole), q and out, the block-table
  entries read and the context lengths.  A physical block shared by several
  sequences counts once ("unique"); the per-sequence sum is the "logical"
  traffic a kernel without reuse would pay.
  With ``kv_int8`` a tile is the INT8 cache's: one-byte codes and one fp32
  scale per token.
* :func:`append_traffic` counts the bytes of one ``paged_kv_append`` call.
"""

from __future__ import annotations

import torch

BLOCK_SIZE = 16


def kv_bytes_per_token(n_layers: int, n_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    return n_layers * 2 * n_kv_heads * head_dim * elem_bytes


def blocks_for(n_tokens: int, block_size: int = BLOCK_SIZE) -> int:
    return (n_tokens + block_size - 1) // block_size


def decode_traffic(block_tables: torch.Tensor, context_lens: torch.Tensor, n_q_heads: int,
                   n_kv_heads: int, head_dim: int, elem_bytes: int,
                   block_size: int = BLOCK_SIZE, kv_int8: bool = False) -> dict:
    """``elem_bytes`` is the element size of q and out; with ``kv_int8`` the
    cache holds one-byte codes plus one fp32 scale per token for K and V."""
    lens = [int(x) for x in context_lens.tolist()]
    bt = block_tables.cpu()
    used = []
    logical_blocks = 0
    for b, n in enumerate(lens):
        nb = blocks_for(n, block_size)
        logical_blocks += nb
        if nb:
            used.append(bt[b, :nb])
    unique_blocks = int(torch.unique(torch.cat(used)).numel()) if used else 0
    # One kv head of one block, K or V (INT8: codes plus a scale per token).
    tile = block_size * (head_dim + 4) if kv_int8 else block_size * head_dim * elem_bytes
    kv_unique = unique_blocks * n_kv_heads * tile * 2
    kv_logical = logical_blocks * n_kv_heads * tile * 2
    batch = len(lens)
    q_out = batch * n_q_heads * head_dim * elem_bytes * 2
    meta = logical_blocks * 4 + batch * 4
    return {
        "unique_blocks": unique_blocks,
        "logical_blocks": logical_blocks,
        "tiles_unique": unique_blocks * n_kv_heads,
        "tile_bytes_kv": 2 * tile,
        "kv_unique": kv_unique,
        "kv_logical": kv_logical,
        "q_out": q_out,
        "meta": meta,
        "total_unique": kv_unique + q_out + meta,
        "total_logical": kv_logical + q_out + meta,
        "tokens": sum(lens),
    }


def append_traffic(num_tokens: int, n_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    row = n_kv_heads * head_dim * elem_bytes
    # read k and v rows and the slot, write both rows into the cache
    return num_tokens * (2 * row + 8 + 2 * row)
