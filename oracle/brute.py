"""Second oracle: pure-Python brute force in 50-digit decimal arithmetic.

Test infrastructure for tiny cases only.  Written independently of the C
oracle: it takes the cache as nested Python lists, walks the block table one
token at a time and evaluates single-query attention (dot products with every
key, a softmax, a weighted sum of the values) with ``decimal`` at 50
significant digits, so that its result is the exact attention output of the
given inputs to far below fp64 resolution.  Inputs are exact binary floats,
which ``Decimal`` represents exactly.

The method followed: "KV Cache and PagedAttention" (gyaansetu), section on the
attention computation (Q of the new token, dot with all K, weights, weighted
sum of V); the block table of "Transformer anatomy" ch. 15 §15.5 (entry i is
the physical block of logical block i, 16 tokens per block).
"""

from __future__ import annotations

from decimal import Decimal, localcontext


def attention_rows(q, k_cache, v_cache, block_tables, context_lens, scale, n_q_heads,
                   n_kv_heads, block_size, prec: int = 50):
    """q: [B][n_q][d] floats; caches: [num_blocks][n_kv][bs][d] floats.
    Returns [B][n_q][d] Python floats (correctly rounded from the decimal result)."""
    group = n_q_heads // n_kv_heads
    out = []
    with localcontext() as ctx:
        ctx.prec = prec
        sc = Decimal(scale)
        for b, qb in enumerate(q):
            n = int(context_lens[b])
            rows = []
            for h in range(n_q_heads):
                kv = h // group
                d = len(qb[h])
                if n == 0:
                    rows.append([0.0] * d)
                    continue
                qh = [Decimal(x) for x in qb[h]]
                keys, vals = [], []
                for t in range(n):
                    blk = int(block_tables[b][t // block_size])
                    keys.append(k_cache[blk][kv][t % block_size])
                    vals.append(v_cache[blk][kv][t % block_size])
                scores = [sc * sum(qh[e] * Decimal(key[e]) for e in range(d)) for key in keys]
                top = max(scores)
                weights = [(s - top).exp() for s in scores]
                total = sum(weights)
                rows.append([float(sum(w * Decimal(v[e]) for w, v in zip(weights, vals)) / total)
                             for e in range(d)])
            out.append(rows)
    return out
