"""INT8 paged KV cache on the GPU through the C ABI: the quantising append
bit for bit against the oracle's append (codes and scales), and the decode
over the INT8 cache against the oracle's fp64 decode over the same codes."""

import pytest
import torch

import oracle
import paged_kv_cache_386_b200 as pkv
import workloads as W
from tests.gpu_helpers import assert_close, bits, sample_rows

pytestmark = pytest.mark.gpu


def _gpu_cache(w):
    """Fill an INT8 cache on the GPU with every cached token of `w` and its
    appended token, through the GPU append."""
    dev = torch.device("cuda")
    cache = W.int8_cache_buffers(w).to(dev)
    kr, vr, slots = W.cached_token_rows(w)
    pkv.paged_kv_append_int8(kr.to(dev), vr.to(dev), slots.to(dev), cache)
    if w.appended:
        pkv.paged_kv_append_int8(w.k_new.to(dev), w.v_new.to(dev), w.slot_mapping.to(dev), cache)
    return cache


def _decode(w, cache):
    dev = torch.device("cuda")
    out = pkv.paged_attention_decode_int8(w.q.to(dev), cache, w.block_tables.to(dev), w.context_lens.to(dev),
                                          w.scale)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_error() == 0
    return out.cpu()


def _check(w, rows=None):
    cache = _gpu_cache(w)
    ref, ocache = oracle.workload_decode_int8(w, rows=rows)
    assert torch.equal(cache.cpu(), ocache), "INT8 records (codes and scale bits) differ from the oracle"
    out = _decode(w, cache)
    return assert_close(out, ref, w.dtype, rows=rows, what=w.name)


SHAPES = [
    (torch.bfloat16, 32, 8),   # G = 4
    (torch.float16, 32, 8),
    (torch.bfloat16, 64, 8),   # G = 8
    (torch.bfloat16, 32, 2),   # G = 16
    (torch.float16, 64, 2),    # G = 32: two 16-row groups per kv head
    (torch.float16, 16, 16),   # G = 1 (MHA) on the tensor cores
    (torch.bfloat16, 12, 4),   # G = 3
]


@pytest.mark.parametrize("dtype,nq,nkv", SHAPES, ids=[f"{str(s[0])[6:]}-{s[1]}x{s[2]}" for s in SHAPES])
def test_int8_decode_head_shapes(dtype, nq, nkv):
    lens = [1, 15, 16, 17, 100, 333, 1024, 47]
    _check(W.build_workload("i8", lens, nq, nkv, 128, dtype, seed=61))


def test_int8_full_size_gqa_sampled():
    w = W.uniform_gqa(seed=0)
    _check(w, rows=sample_rows(w, 96))


def test_int8_full_size_mha_sampled():
    w = W.lognormal_mha(seed=0)
    _check(w, rows=sample_rows(w, 96))


@pytest.mark.parametrize("src", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
def test_int8_append_bit_exact(src, d):
    g = torch.Generator().manual_seed(62)
    n, n_kv, nb = 40, 4, 6
    k = (torch.randn((n, n_kv, d), generator=g) * torch.rand((n, 1, 1), generator=g) * 5).to(src)
    v = (torch.randn((n, n_kv, d), generator=g) * 3).to(src)
    k[3] = 0                                                    # all-zero rows: scale 0, codes 0
    slots = torch.randperm(nb * 16, generator=g)[:n].to(torch.int64)
    slots[5] = -1                                               # padding token: skipped
    ocache = torch.zeros((nb, n_kv, 32 * d + 128), dtype=torch.uint8)
    ocache[:, :, 32 * d:].view(torch.float32).fill_(float("nan"))
    cache = ocache.clone().cuda()
    oracle.kv_append_int8(k, v, slots, ocache)
    pkv.paged_kv_append_int8(k.cuda(), v.cuda(), slots.cuda(), cache)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_error() == 0
    assert torch.equal(cache.cpu(), ocache)


def test_int8_placement_bit_exact_and_deterministic():
    w = W.uniform_gqa(batch=8, len_lo=30, len_hi=1200, seed=63)
    cache = _gpu_cache(w)
    a = _decode(w, cache)
    assert torch.equal(bits(a), bits(_decode(w, cache)))
    # The same tokens with every physical block moved elsewhere.
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(5))
    dev = torch.device("cuda")
    moved = torch.empty_like(cache)
    moved[perm.to(dev)] = cache
    m = W.uniform_gqa(batch=8, len_lo=30, len_hi=1200, seed=63)
    m.block_tables = torch.where(w.block_tables >= 0, perm[w.block_tables.clamp(min=0).long()].int(), w.block_tables)
    b = _decode(m, moved)
    assert torch.equal(bits(a), bits(b))


def test_int8_empty_and_unsupported():
    w = W.build_workload("i8e", [5, 40], 8, 2, 128, torch.bfloat16, seed=64, append=False)
    w.context_lens[0] = 0
    cache = _gpu_cache(w)
    out = _decode(w, cache)
    assert torch.equal(out[0], torch.zeros_like(out[0]))
    ref, _ = oracle.workload_decode_int8(w)
    assert_close(out, ref, w.dtype, what="i8 empty")
    dev = torch.device("cuda")
    with pytest.raises(pkv.PagedKVError) as e:   # fp32 queries are not supported on the INT8 cache
        pkv.paged_attention_decode_int8(w.q.float().to(dev), cache, w.block_tables.to(dev),
                                        w.context_lens.to(dev), w.scale)
    assert e.value.status == 2
