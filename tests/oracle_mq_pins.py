"""Pins of the oracle's multi-query decode (q_len new tokens per sequence,
causal among them), against facts that do not come from the oracle itself:
torch scaled_dot_product_attention in fp64 with an explicit causal mask on
the gathered keys and values, and the single-query decode for q_len = 1."""

from __future__ import annotations

import torch

import oracle
from workloads import build_workload


def _gather(w, kc, vc, b):
    bs = w.block_size
    n = int(w.context_lens[b])
    rows = [(int(w.block_tables[b, j // bs]), j % bs) for j in range(n)]
    K = torch.stack([kc[p, :, o] for p, o in rows], dim=1).double()   # [n_kv, n, d]
    V = torch.stack([vc[p, :, o] for p, o in rows], dim=1).double()
    return K, V


def pin_mq_equals_causal_sdpa(lib):
    for dtype, nq, nkv, q_len in ((torch.bfloat16, 8, 2, 3), (torch.float16, 4, 4, 5), (torch.float32, 6, 3, 1)):
        w = build_workload("mq", [5, 16, 17, 40, 9], nq, nkv, 64, dtype, seed=71, q_len=q_len)
        out, kc, vc = oracle.workload_decode_mq(w, lib=lib)
        G = nq // nkv
        q4 = w.q if w.q.dim() == 4 else w.q.unsqueeze(1)
        for b in range(w.batch):
            K, V = _gather(w, kc, vc, b)
            n = K.shape[1]
            pos = torch.arange(n - q_len, n)
            mask = torch.arange(n)[None, :] <= pos[:, None]                       # [q_len, n]
            q = q4[b].double().permute(1, 0, 2).reshape(nkv, G, q_len, -1)        # [n_kv, G, q_len, d]
            ref = torch.nn.functional.scaled_dot_product_attention(q, K[:, None], V[:, None], attn_mask=mask,
                                                                   scale=w.scale)
            ref = ref.reshape(nq, q_len, -1).permute(1, 0, 2)                     # [q_len, n_q, d]
            err = (out[b] - ref).abs().max().item()
            assert err < 1e-12, (dtype, b, err)


def pin_mq_single_query_case(lib):
    w = build_workload("mq1", [7, 33, 1, 64], 8, 2, 128, torch.bfloat16, seed=72)
    a, _, _ = oracle.workload_decode(w, lib=lib)
    b, _, _ = oracle.workload_decode_mq(w, lib=lib)
    assert torch.equal(a, b[:, 0])


def pin_mq_rejects_short_context(lib):
    w = build_workload("mqs", [6, 10], 4, 2, 64, torch.float16, seed=73, q_len=4)
    w.context_lens[0] = 3
    try:
        oracle.workload_decode_mq(w, lib=lib)
    except oracle.OracleError:
        return
    raise AssertionError("context shorter than q_len accepted")


PINS = [pin_mq_equals_causal_sdpa, pin_mq_single_query_case, pin_mq_rejects_short_context]
