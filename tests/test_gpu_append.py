"""GPU paged_kv_append against the oracle's append: bit-exact, canaries kept,
padding slots skipped, out-of-range slots flagged and skipped."""

import pytest
import torch

import oracle
import paged_kv_cache_386_b200 as pkv
from tests.gpu_helpers import bits

pytestmark = pytest.mark.gpu


def _canary(shape, dtype):
    t = torch.empty(shape, dtype=dtype)
    t.view(torch.int32 if dtype == torch.float32 else torch.int16).fill_(0x7A5C)
    return t


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("n_kv,d", [(1, 64), (8, 128), (32, 128)])
def test_append_bit_exact(dtype, n_kv, d):
    num_blocks, bs = 97, 16
    g = torch.Generator().manual_seed(n_kv * 1000 + d)
    n_tok = 300
    slots = torch.randperm(num_blocks * bs, generator=g)[:n_tok].to(torch.int64)
    slots[::17] = -1   # padding tokens
    k = torch.randn(n_tok, n_kv, d, generator=g).to(dtype)
    v = torch.randn(n_tok, n_kv, d, generator=g).to(dtype)
    kc, vc = _canary((num_blocks, n_kv, bs, d), dtype), _canary((num_blocks, n_kv, bs, d), dtype)
    okc, ovc = kc.clone(), vc.clone()
    oracle.kv_append(k, v, slots, okc, ovc, bs)
    gkc, gvc = kc.cuda(), vc.cuda()
    pkv.paged_kv_append(k.cuda(), v.cuda(), slots.cuda(), gkc, gvc)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_error() == 0
    assert torch.equal(bits(gkc.cpu()), bits(okc)) and torch.equal(bits(gvc.cpu()), bits(ovc))


def test_append_out_of_range_slot_is_flagged_and_skipped():
    num_blocks, n_kv, bs, d = 4, 2, 16, 64
    kc = _canary((num_blocks, n_kv, bs, d), torch.bfloat16)
    k = torch.randn(3, n_kv, d).to(torch.bfloat16)
    slots = torch.tensor([5, num_blocks * bs, 63], dtype=torch.int64)
    okc, ovc = kc.clone(), kc.clone()
    oracle.kv_append(k[[0, 2]], k[[0, 2]], slots[[0, 2]], okc, ovc, bs)
    gkc, gvc = kc.cuda(), kc.clone().cuda()
    pkv.paged_kv_append(k.cuda(), k.cuda(), slots.cuda(), gkc, gvc)
    torch.cuda.synchronize()
    assert pkv.pkv_get_device_error() & pkv.DEVERR_SLOT
    assert torch.equal(bits(gkc.cpu()), bits(okc))


def test_append_on_a_side_stream_is_ordered_before_decode():
    from workloads import uniform_gqa
    from tests.gpu_helpers import assert_close
    w = uniform_gqa(batch=4, len_lo=20, len_hi=300, seed=31)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        kc, vc = w.k_cache.cuda(), w.v_cache.cuda()
        pkv.paged_kv_append(w.k_new.cuda(), w.v_new.cuda(), w.slot_mapping.cuda(), kc, vc, stream=s)
        out = pkv.paged_attention_decode(w.q.cuda(), kc, vc, w.block_tables.cuda(), w.context_lens.cuda(),
                                         w.scale, stream=s)
    s.synchronize()
    ref, _, _ = oracle.workload_decode(w)
    assert_close(out.cpu(), ref, w.dtype, what="side stream")
