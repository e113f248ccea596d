"""paged_attention_decode_noalloc, called through the C ABI, against
paged_attention_decode on the same inputs.

The no-allocation entry point is for callers that cannot allocate device
memory (a plugin whose host framework owns all device memory, a serving loop
that must never call an allocator on its hot path, a process whose free
memory all went to its KV pool).  Its split-context scratch is one static
device array shared by every call, which keeps the previous call's contents;
so the test makes two calls in a row on different problems and checks each
against the allocating entry point within the parity tolerances."""

import pytest
import torch

import paged_kv_cache_386_b200 as pkv
import workloads as W
from tests.gpu_helpers import TOL, errors

pytestmark = pytest.mark.gpu


def _both(w):
    dev = torch.device("cuda")
    kc, vc = w.k_cache.to(dev), w.v_cache.to(dev)
    pkv.paged_kv_append(w.k_new.to(dev), w.v_new.to(dev), w.slot_mapping.to(dev), kc, vc)
    q, bt, cl = w.q.to(dev), w.block_tables.to(dev), w.context_lens.to(dev)
    ref = torch.empty_like(q)
    got = torch.empty_like(q)
    pkv.paged_attention_decode(q, kc, vc, bt, cl, w.scale, out=ref)
    pkv.paged_attention_decode_noalloc(q, kc, vc, bt, cl, w.scale, out=got)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_error() == 0
    return got.cpu(), ref.cpu()


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    first = W.uniform_gqa(batch=24, len_lo=100, len_hi=4000, seed=41)            # GQA, tensor cores, splits
    second = W.build_workload("mha_f16", [1, 9, 300, 2000, 17], 16, 16, 64,      # MHA, CUDA cores, other sizes
                              torch.float16, seed=42)
    for w in (first, second):
        got, ref = _both(w)
        e = errors(got, ref.double())
        tol = TOL[w.dtype]
        assert e["finite"]
        assert e["max_abs"] <= tol["max_abs"] and e["rel_l2"] <= tol["rel_l2"], (w.name, e)
