"""paged_attention_decode_noalloc, called through the C ABI, against
paged_attention_decode on the same inputs.

The no-allocation entry point is for callers that cannot allocate device
memory (a plugin whose host framework owns all device memory, a serving loop
that must never call an allocator on its hot path, a process whose free
memory all went to its KV pool).  Its split-context scratch is one static
device array shared by every call, which keeps the previous call's contents.
The header promises results bit-identical to paged_attention_decode with its
default split, so the test makes two calls in a row on different problems --
the second one smaller, so that scratch left by the first would show -- and
compares each with the allocating entry point bit for bit."""

import pytest
import torch

import paged_kv_cache_386_b200 as pkv
import workloads as W
from tests.gpu_helpers import bits

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


def test_noalloc_matches_decode_bit_for_bit_on_two_calls_in_a_row():
    first = W.uniform_gqa(batch=24, len_lo=100, len_hi=4000, seed=41)            # GQA, tensor cores, splits
    second = W.build_workload("mha_f16", [1, 9, 300, 700, 17], 16, 16, 64,       # MHA, CUDA cores, fewer rows
                              torch.float16, seed=42)
    for w in (first, second):
        got, ref = _both(w)
        assert torch.isfinite(got.double()).all(), w.name
        assert torch.equal(bits(got), bits(ref)), w.name


def test_noalloc_checks_arguments_before_anything_runs():
    w = W.build_workload("bad", [20, 40], 4, 4, 64, torch.bfloat16, seed=43)
    dev = torch.device("cuda")
    kc = w.k_cache.to(dev)
    with pytest.raises(ValueError):   # out of another dtype is refused by the binding
        pkv.paged_attention_decode_noalloc(w.q.to(dev), kc, kc, w.block_tables.to(dev), w.context_lens.to(dev),
                                           w.scale, out=torch.empty(w.q.shape, dtype=torch.float16, device=dev))
