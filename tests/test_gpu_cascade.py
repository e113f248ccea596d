"""Cascade decode (shared prefix attended once per group and kv head, then the
private suffixes) against the CPU oracle on the full, concatenated tables."""

import pytest
import torch

import oracle
import paged_kv_cache_386_b200 as pkv
import workloads as W
from tests.gpu_helpers import assert_close, bits, drop_blocks, sample_rows

pytestmark = pytest.mark.gpu


def run_cascade(w, cv=None, check_errors=True, workspace=None, **opts):
    dev = torch.device("cuda")
    kc, vc = w.k_cache.to(dev), w.v_cache.to(dev)
    if w.appended:
        pkv.paged_kv_append(w.k_new.to(dev), w.v_new.to(dev), w.slot_mapping.to(dev), kc, vc)
    cv = cv or W.cascade_view(w)
    out = pkv.paged_attention_decode_cascade(
        w.q.to(dev), kc, vc, cv.prefix_block_tables.to(dev), cv.prefix_lens.to(dev), cv.seq_group.to(dev),
        cv.block_tables.to(dev), cv.context_lens.to(dev), w.scale, workspace=workspace, **opts)
    torch.cuda.synchronize()
    if check_errors:
        assert pkv.pkv_get_device_error() == 0
    return out.cpu()


def check(w, rows=None):
    out = run_cascade(w)
    ref, _, _ = oracle.workload_decode(w, rows=rows)
    return assert_close(out, ref, w.dtype, rows=rows, what=w.name)


SMALL = {
    "shared_prefix_small": lambda: W.shared_prefix(n_seqs=12, prefix=512, seed=41),
    "best_of_8_small": lambda: W.best_of_n(prompts=3, n=8, seed=42),
    "prefix_ragged_tile": lambda: W.shared_prefix(n_seqs=5, prefix=272, suffix=(16, 100), seed=43),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_cascade_small_full_output(name):
    check(SMALL[name]())


@pytest.mark.parametrize("name", ["shared_prefix_70b", "best_of_8"])
def test_cascade_full_size_sampled(name):
    w = W.shared_prefix(seed=0) if name == "shared_prefix_70b" else W.best_of_n(seed=0)
    check(w, rows=sample_rows(w, 128))


SHAPES = [
    (torch.bfloat16, 128, 8, 8),     # G=1: CUDA-core suffix path continues from the prefix state
    (torch.float16, 64, 16, 4),      # G=4, d=64
    (torch.bfloat16, 128, 32, 2),    # G=16: 16-row tensor-core tiles
    (torch.bfloat16, 128, 40, 4),    # G=10
]


@pytest.mark.parametrize("dtype,d,nq,nkv", SHAPES, ids=[f"{str(s[0])[6:]}-d{s[1]}-{s[2]}x{s[3]}" for s in SHAPES])
def test_cascade_head_shapes(dtype, d, nq, nkv):
    lens = [160 + 5, 160 + 40, 160 + 1, 160 + 77, 160 + 16]
    w = W.build_workload("cshape", lens, nq, nkv, d, dtype, seed=44, groups=[([0, 1, 2, 3, 4], 160)])
    check(w)


def test_cascade_mixed_groups_and_loners():
    lens = [96 + 10, 300, 96 + 33, 64 + 5, 64 + 70, 50, 96 + 1]
    w = W.build_workload("mixed", lens, 16, 2, 128, torch.bfloat16, seed=45,
                         groups=[([0, 2, 6], 96), ([3, 4], 64)])
    cv = W.cascade_view(w)
    assert cv.seq_group.tolist() == [0, -1, 0, 1, 1, -1, 0]
    check(w)


def test_cascade_empty_suffix_and_empty_prefix():
    w = W.build_workload("edges", [64 + 20, 64 + 3, 48 + 9], 8, 2, 128, torch.bfloat16, seed=46, append=False,
                         groups=[([0, 1], 64), ([2], 48)])
    w.context_lens[1] = 64          # sequence 1 is exactly the shared prefix
    cv = W.cascade_view(w)
    assert int(cv.context_lens[1]) == 0
    cv.prefix_lens[1] = 0           # group 1: no shared tokens after all
    wide = torch.full((w.batch, w.max_blocks_per_seq), -1, dtype=torch.int32)
    wide[:, : cv.block_tables.shape[1]] = cv.block_tables
    wide[2] = w.block_tables[2]     # its suffix is then its whole context
    cv.block_tables = wide
    cv.context_lens[2] = w.context_lens[2]
    out = run_cascade(w, cv)
    ref, _, _ = oracle.workload_decode(w)
    assert_close(out, ref, w.dtype, what="edges")


def test_cascade_matches_plain_decode():
    w = W.shared_prefix(n_seqs=8, prefix=256, seed=47)
    out_c = run_cascade(w)
    dev = torch.device("cuda")
    kc, vc = w.k_cache.to(dev), w.v_cache.to(dev)
    pkv.paged_kv_append(w.k_new.to(dev), w.v_new.to(dev), w.slot_mapping.to(dev), kc, vc)
    out_p = pkv.paged_attention_decode(w.q.to(dev), kc, vc, w.block_tables.to(dev), w.context_lens.to(dev),
                                       w.scale).cpu()
    assert_close(out_c, out_p.double(), w.dtype, what="cascade vs plain")
    assert torch.equal(bits(run_cascade(w)), bits(out_c))   # deterministic


def test_cascade_bad_group_id_sets_flag():
    w = W.shared_prefix(n_seqs=4, prefix=64, seed=48)
    cv = W.cascade_view(w)
    cv.seq_group[2] = 5   # no such group
    run_cascade(w, cv, check_errors=False)
    assert pkv.pkv_get_device_error() & pkv.DEVERR_CONTEXT


def test_cascade_fp32_is_unsupported():
    w = W.build_workload("f32", [40, 50], 4, 2, 64, torch.float32, seed=49, groups=[([0, 1], 32)])
    with pytest.raises(pkv.PagedKVError) as e:
        run_cascade(w)
    assert e.value.status == 2


# Prefix lengths that leave some cluster ranks with no stage (16 tokens: one
# 64-key stage), end in a partial stage (272, 336) or split unevenly (592:
# ten stages over 3 or 4 ranks), with a ragged last row tile.
SPLIT_PREFIXES = [16, 272, 336, 592]


@pytest.mark.parametrize("splits", [1, 2, 3, 4])
@pytest.mark.parametrize("prefix", SPLIT_PREFIXES)
def test_cascade_prefix_split_across_cluster(splits, prefix):
    w = W.shared_prefix(n_seqs=18, prefix=prefix, suffix=(1, 60), seed=50 + prefix)
    out = run_cascade(w, prefix_splits=splits, prefix_kernel=1)
    ref, _, _ = oracle.workload_decode(w)
    assert_close(out, ref, w.dtype, what=f"splits={splits} prefix={prefix}")


@pytest.mark.parametrize("kernel", [1, 2])
def test_cascade_both_prefix_kernels(kernel):
    w = W.best_of_n(prompts=3, n=8, prompt_len=384, gen_len=40, seed=51)
    out = run_cascade(w, prefix_kernel=kernel)
    ref, _, _ = oracle.workload_decode(w)
    assert_close(out, ref, w.dtype, what=f"prefix kernel {kernel}")


def test_cascade_split_full_size_sampled():
    w = W.shared_prefix(seed=1)
    rows = sample_rows(w, 96)
    for splits in (2, 4):
        out = run_cascade(w, prefix_splits=splits)
        ref, _, _ = oracle.workload_decode(w, rows=rows)
        assert_close(out, ref, w.dtype, rows=rows, what=f"shared_prefix_70b splits={splits}")


@pytest.mark.parametrize("scale", [-0.0884, 0.0, 0.5])
@pytest.mark.parametrize("kernel", [1, 2])
def test_cascade_scale_sign_and_size(scale, kernel):
    # A negative scale runs on -Q in the tensor-memory kernel; zero gives
    # uniform weights; a large one stresses the lazy rescale of O.
    w = W.shared_prefix(n_seqs=10, prefix=208, suffix=(1, 40), seed=53, scale=scale)
    out = run_cascade(w, prefix_kernel=kernel, prefix_splits=2 if kernel == 1 else 0)
    ref, _, _ = oracle.workload_decode(w)
    assert_close(out, ref, w.dtype, what=f"scale={scale} kernel={kernel}")


@pytest.mark.parametrize("splits", [1, 2])
def test_cascade_fp16_tensor_memory_kernel(splits):
    w = W.shared_prefix(n_seqs=9, prefix=400, suffix=(1, 70), dtype=torch.float16, seed=54)
    out = run_cascade(w, prefix_kernel=1, prefix_splits=splits)
    ref, _, _ = oracle.workload_decode(w)
    assert_close(out, ref, w.dtype, what=f"fp16 splits={splits}")


# Out-of-range ids in a shared prefix table: both prefix kernels copy nothing
# useful for those blocks, mask their keys and set the flag; the result is
# attention over the remaining tokens (the oracle without those blocks).
@pytest.mark.parametrize("kernel,splits", [(1, 1), (1, 2), (2, 0)])
def test_cascade_bad_prefix_block_is_left_out(kernel, splits):
    w = W.shared_prefix(n_seqs=6, prefix=256, suffix=(10, 80), seed=55)
    cv = W.cascade_view(w)
    drop = [2, 9, 15]   # inside the first stage, inside a later one, the prefix's last block
    ref, _, _ = oracle.workload_decode(drop_blocks(w, {b: drop for b in range(w.batch)}))
    cv.prefix_block_tables[0, 2] = w.num_blocks
    cv.prefix_block_tables[0, 9] = -1
    cv.prefix_block_tables[0, 15] = 1 << 30
    out = run_cascade(w, cv, check_errors=False, prefix_kernel=kernel, prefix_splits=splits)
    assert pkv.pkv_get_device_error() & pkv.DEVERR_BLOCK_ID
    assert_close(out, ref, w.dtype, what=f"bad prefix blocks, kernel {kernel}")


def test_cascade_repeated_full_size_runs_are_bit_identical():
    # Every run of the same inputs gives the same bits.  A wait that passed
    # before a set's last P V had finished once left about one full-size run
    # in fifty with a wrong 128-row tile; sixty runs over three split counts
    # catch such a race with high probability.  One run is also checked
    # against the oracle on sampled rows.
    w = W.shared_prefix(seed=3)
    dev = torch.device("cuda")
    kc, vc = w.k_cache.to(dev), w.v_cache.to(dev)
    pkv.paged_kv_append(w.k_new.to(dev), w.v_new.to(dev), w.slot_mapping.to(dev), kc, vc)
    cv = W.cascade_view(w)
    args = [t.to(dev) for t in (cv.prefix_block_tables, cv.prefix_lens, cv.seq_group, cv.block_tables,
                                cv.context_lens)]
    q = w.q.to(dev)
    rows = sample_rows(w, 48)
    ref, _, _ = oracle.workload_decode(w, rows=rows)
    for splits in (0, 2, 4):
        first = None
        for _ in range(20):
            out = pkv.paged_attention_decode_cascade(q, kc, vc, *args, w.scale, prefix_splits=splits)
            if first is None:
                first = out.clone()
            else:
                assert torch.equal(bits(out), bits(first)), f"splits={splits}: runs differ"
        torch.cuda.synchronize()
        assert pkv.pkv_get_device_error() == 0
        assert_close(first.cpu(), ref, w.dtype, rows=rows, what=f"repeated runs, splits={splits}")
