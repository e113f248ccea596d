"""paged_kv_append_and_decode (the append fused into the decode launch),
called through the C ABI: it must give the cache and the output of
paged_kv_append followed by paged_attention_decode bit for bit, and match the
oracle within the parity tolerances."""

import pytest
import torch

import oracle
import paged_kv_cache_386_b200 as pkv
import workloads as W
from tests.gpu_helpers import assert_close, bits, sample_rows

pytestmark = pytest.mark.gpu


def _inputs(w):
    dev = torch.device("cuda")
    return (w.q.to(dev), w.k_new.to(dev), w.v_new.to(dev), w.slot_mapping.to(dev), w.k_cache.to(dev),
            w.v_cache.to(dev), w.block_tables.to(dev), w.context_lens.to(dev))


def fused(w, **kw):
    q, k, v, sl, kc, vc, bt, cl = _inputs(w)
    out = pkv.paged_kv_append_and_decode(q, k, v, sl, kc, vc, bt, cl, w.scale, **kw)
    torch.cuda.synchronize()
    return out.cpu(), kc.cpu(), vc.cpu()


def separate(w):
    q, k, v, sl, kc, vc, bt, cl = _inputs(w)
    pkv.paged_kv_append(k, v, sl, kc, vc)
    out = pkv.paged_attention_decode(q, kc, vc, bt, cl, w.scale)
    torch.cuda.synchronize()
    return out.cpu(), kc.cpu(), vc.cpu()


CASES = {
    "tiny_mha_f32": lambda: W.tiny_mha(seed=0),
    "llama3_8b_gqa_small": lambda: W.uniform_gqa(batch=12, len_lo=128, len_hi=1500, seed=61),
    "llama2_7b_mha_small": lambda: W.lognormal_mha(batch=48, seed=62),
    "long_ctx_small": lambda: W.long_context(batch=2, ctx=12000, seed=63),
    "gqa16_f16_d64": lambda: W.build_workload("g16", [1, 16, 17, 400, 1023], 32, 2, 64, torch.float16, seed=64),
    "fp32_gqa": lambda: W.build_workload("f32", [1, 5, 33, 300], 8, 2, 128, torch.float32, seed=65),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fused_equals_separate_calls_and_the_oracle(name):
    w = CASES[name]()
    out_f, kc_f, vc_f = fused(w)
    assert pkv.pkv_get_device_error() == 0
    out_s, kc_s, vc_s = separate(w)
    assert torch.equal(bits(kc_f), bits(kc_s)) and torch.equal(bits(vc_f), bits(vc_s)), "cache differs"
    assert torch.equal(bits(out_f), bits(out_s)), "output differs from append + decode"
    ref, okc, ovc = oracle.workload_decode(w)
    assert torch.equal(bits(kc_f), bits(okc)) and torch.equal(bits(vc_f), bits(ovc)), "append not bit-exact"
    assert_close(out_f, ref, w.dtype, what=name)


@pytest.mark.parametrize("name", ["long_ctx_128k", "llama3_8b_gqa"])
def test_fused_full_size(name):
    w = W.long_context(seed=0) if name == "long_ctx_128k" else W.uniform_gqa(seed=0)
    out_f, kc_f, vc_f = fused(w)
    assert pkv.pkv_get_device_error() == 0
    out_s, _, _ = separate(w)
    assert torch.equal(bits(out_f), bits(out_s))
    rows = sample_rows(w, 64)
    ref, okc, ovc = oracle.workload_decode(w, rows=rows)
    assert torch.equal(bits(kc_f), bits(okc)) and torch.equal(bits(vc_f), bits(ovc))
    assert_close(out_f, ref, w.dtype, rows=rows, what=name)


def test_fused_skips_padding_and_flags_a_slot_beyond_the_pool():
    w = W.uniform_gqa(batch=6, len_lo=40, len_hi=300, seed=66)
    w.slot_mapping[2] = -1                       # padding: nothing written for token 2
    w.slot_mapping[4] = w.num_blocks * 16 + 3    # beyond the pool: skipped and flagged
    out_f, kc_f, vc_f = fused(w)
    assert pkv.pkv_get_device_error() & pkv.DEVERR_SLOT
    out_s, kc_s, vc_s = separate(w)
    assert pkv.pkv_get_device_error() & pkv.DEVERR_SLOT
    assert torch.equal(bits(kc_f), bits(kc_s)) and torch.equal(bits(vc_f), bits(vc_s))
    assert torch.equal(bits(out_f), bits(out_s))


def test_fused_with_no_tokens_is_the_plain_decode_and_with_no_batch_the_append():
    w = W.uniform_gqa(batch=5, len_lo=40, len_hi=900, seed=67, )
    q, k, v, sl, kc, vc, bt, cl = _inputs(w)
    pkv.paged_kv_append(k, v, sl, kc, vc)
    ref = pkv.paged_attention_decode(q, kc, vc, bt, cl, w.scale)
    out = pkv.paged_kv_append_and_decode(q, k[:0], v[:0], sl[:0], kc, vc, bt, cl, w.scale)
    assert torch.equal(bits(out.cpu()), bits(ref.cpu()))
    # batch 0: the append alone
    _, k, v, sl, kc2, vc2, _, _ = _inputs(w)
    pkv.paged_kv_append_and_decode(q[:0], k, v, sl, kc2, vc2, bt[:0], cl[:0], w.scale)
    torch.cuda.synchronize()
    assert torch.equal(bits(kc2.cpu()), bits(kc.cpu())) and torch.equal(bits(vc2.cpu()), bits(vc.cpu()))
