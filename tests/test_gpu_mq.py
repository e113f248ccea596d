"""Several queries per sequence (the last q_len tokens of each context,
causal among themselves) through the C ABI, against the oracle's fp64
multi-query decode on the same seeded inputs."""

import pytest
import torch

import oracle
import paged_kv_cache_386_b200 as pkv
import workloads as W
from tests.gpu_helpers import assert_close, bits

pytestmark = pytest.mark.gpu


def run_mq(w, check_errors=True, workspace=None):
    dev = torch.device("cuda")
    kc, vc = w.k_cache.to(dev), w.v_cache.to(dev)
    pkv.paged_kv_append(w.k_new.to(dev), w.v_new.to(dev), w.slot_mapping.to(dev), kc, vc)
    q = w.q if w.q.dim() == 4 else w.q.unsqueeze(1)
    out = pkv.paged_attention_decode_mq(q.contiguous().to(dev), kc, vc, w.block_tables.to(dev),
                                        w.context_lens.to(dev), w.scale, workspace=workspace)
    torch.cuda.synchronize()
    if check_errors:
        assert pkv.pkv_get_device_error() == 0
    return out.cpu()


def check(w):
    out = run_mq(w)
    ref, _, _ = oracle.workload_decode_mq(w)
    return assert_close(out, ref, w.dtype, what=f"{w.name} q_len={w.q_len}")


CASES = [
    # dtype, n_q, n_kv, d, q_len   (rows per segment = heads x queries <= 16)
    (torch.bfloat16, 32, 8, 128, 2),   # G 4: 8 rows (the residual rows stay unused)
    (torch.bfloat16, 32, 8, 128, 3),   # 12 rows
    (torch.bfloat16, 32, 8, 128, 4),   # 16 rows
    (torch.float16, 64, 8, 128, 2),    # G 8: 16 rows
    (torch.bfloat16, 32, 32, 128, 5),  # MHA: 5 rows
    (torch.bfloat16, 32, 2, 64, 4),    # G 16: 4 heads x 4 queries, d 64
    (torch.float16, 32, 8, 64, 16),    # 16 queries: one head x 16 rows
    (torch.bfloat16, 24, 8, 128, 7),   # G 3 with 7 queries: 2 heads would be 14 rows, so 1 head x 7
]


@pytest.mark.parametrize("dtype,nq,nkv,d,q_len", CASES,
                         ids=[f"{str(c[0])[6:]}-{c[1]}x{c[2]}-d{c[3]}-q{c[4]}" for c in CASES])
def test_mq_matches_oracle(dtype, nq, nkv, d, q_len):
    lens = [q_len, q_len + 1, 16, 17, 33, 100, 500, 1500]
    check(W.build_workload("mq", lens, nq, nkv, d, dtype, seed=81 + q_len, q_len=q_len))


def test_mq_llama3_8b_shape_verify_four_drafts():
    w = W.uniform_gqa(batch=32, seed=82, q_len=4)
    check(w)


def test_mq_deterministic_and_q_len_one_equals_decode():
    w = W.build_workload("mq1", [40, 300, 1000, 7], 32, 8, 128, torch.bfloat16, seed=83, q_len=3)
    assert torch.equal(bits(run_mq(w)), bits(run_mq(w)))
    s = W.build_workload("mq1", [40, 300, 1000, 7], 32, 8, 128, torch.bfloat16, seed=84)
    a = run_mq(s)[:, 0]
    dev = torch.device("cuda")
    kc, vc = s.k_cache.to(dev), s.v_cache.to(dev)
    pkv.paged_kv_append(s.k_new.to(dev), s.v_new.to(dev), s.slot_mapping.to(dev), kc, vc)
    b = pkv.paged_attention_decode(s.q.to(dev), kc, vc, s.block_tables.to(dev), s.context_lens.to(dev), s.scale)
    ref, _, _ = oracle.workload_decode(s)
    assert_close(a, ref, s.dtype, what="q_len 1")
    assert_close(b.cpu(), ref, s.dtype, what="decode")


def test_mq_short_context_is_flagged_and_zero():
    w = W.build_workload("mqs", [8, 40], 8, 2, 128, torch.bfloat16, seed=85, q_len=4)
    w.context_lens[0] = 2                     # fewer tokens than queries
    out = run_mq(w, check_errors=False)
    assert pkv.pkv_get_device_error() & pkv.DEVERR_CONTEXT
    assert torch.equal(out[0], torch.zeros_like(out[0]))
    w.context_lens[0] = 8
    ref, _, _ = oracle.workload_decode_mq(w)
    assert_close(out[1:], ref[1:], w.dtype, what="other sequence")


def test_mq_rejects_fp32_and_long_q():
    w = W.build_workload("mqr", [20], 4, 2, 64, torch.float32, seed=86, q_len=2)
    with pytest.raises(pkv.PagedKVError) as e:
        run_mq(w)
    assert e.value.status == 2
