"""GPU parity of paged_kv_append + paged_attention_decode against the CPU
oracle (called through the C-ABI), on the five workload shapes, their edge
cases and the invariants the method fixes."""

import pytest
import torch

import oracle
import paged_kv_cache_386_b200 as pkv
import workloads as W
from tests.gpu_helpers import assert_close, bits, check_workload, drop_blocks, run_gpu, sample_rows

pytestmark = pytest.mark.gpu


# --- the five shapes at sizes the oracle finishes in seconds (full output) ---

SCALED = {
    "tiny_mha_f32": lambda: W.tiny_mha(seed=0),
    "llama3_8b_gqa_small": lambda: W.uniform_gqa(batch=12, len_lo=128, len_hi=1500, seed=1),
    "llama2_7b_mha_small": lambda: W.lognormal_mha(batch=48, seed=2),
    "shared_prefix_small": lambda: W.shared_prefix(n_seqs=12, prefix=512, seed=3),
    "best_of_8_small": lambda: W.best_of_n(prompts=2, n=8, seed=4),
    "long_ctx_small": lambda: W.long_context(batch=2, ctx=12000, seed=5),
}


@pytest.mark.parametrize("name", list(SCALED))
def test_scaled_configs_full_output(name):
    check_workload(SCALED[name]())


# --- the full-size shapes, on sampled output rows ---

FULL = {
    "llama3_8b_gqa": lambda: W.uniform_gqa(seed=0),
    "llama2_7b_mha": lambda: W.lognormal_mha(seed=0),
    "shared_prefix_70b": lambda: W.shared_prefix(seed=0),
    "best_of_8": lambda: W.best_of_n(seed=0),
    "long_ctx_128k": lambda: W.long_context(seed=0),
}


# Rows compared with the oracle: every row of the long-context shape (4 x 64;
# each of its 46-piece split contexts is then checked in full), 512 of the
# Llama-3-8B and Llama-2-7B shapes, 128 of the shared-prefix ones.
FULL_ROWS = {"long_ctx_128k": None, "llama3_8b_gqa": 512, "llama2_7b_mha": 512,
             "shared_prefix_70b": 128, "best_of_8": 128}


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_configs_sampled(name):
    w = FULL[name]()
    n = FULL_ROWS[name]
    check_workload(w, rows=None if n is None else sample_rows(w, n))


# --- head shapes, dtypes, paths ---

SHAPES = [
    # dtype, head_dim, n_q, n_kv      (group size -> path)
    (torch.bfloat16, 128, 8, 8),      # G=1  CUDA cores
    (torch.float16, 64, 4, 4),        # G=1  CUDA cores, d=64
    (torch.bfloat16, 128, 4, 2),      # G=2  tensor cores
    (torch.float16, 128, 12, 4),      # G=3  tensor cores, odd group
    (torch.bfloat16, 64, 16, 2),      # G=8  tensor cores, d=64
    (torch.float16, 128, 32, 2),      # G=16 tensor cores, 16 rows
    (torch.bfloat16, 128, 64, 2),     # G=32 two segments per kv head
    (torch.bfloat16, 128, 20, 2),     # G=10 16-row tile, 10 used
    (torch.float32, 128, 8, 2),       # fp32 GQA on CUDA cores
    (torch.float32, 64, 6, 3),        # fp32 GQA, d=64
]


@pytest.mark.parametrize("dtype,d,nq,nkv", SHAPES, ids=[f"{str(s[0])[6:]}-d{s[1]}-{s[2]}x{s[3]}" for s in SHAPES])
def test_head_shapes(dtype, d, nq, nkv):
    lens = [1, 5, 16, 17, 31, 32, 33, 250, 700, 1023]
    w = W.build_workload("shape", lens, nq, nkv, d, dtype, seed=11)
    check_workload(w)


def test_cuda_core_path_on_gqa_matches_oracle():
    w = W.uniform_gqa(batch=6, len_lo=16, len_hi=900, seed=12)
    check_workload(w, force_simt=True)


# --- invariants ---

def test_split_count_invariance():
    w = W.uniform_gqa(batch=10, len_lo=100, len_hi=3000, seed=13)
    ref, _, _ = oracle.workload_decode(w)
    outs = {}
    for units in (1, 2, 7, 64, 0, 100000):   # 100000 is capped at 8 units per SM
        outs[units] = run_gpu(w, num_units=units)
        assert_close(outs[units], ref, w.dtype, what=f"units={units}")
    # Same split -> same bits.
    assert torch.equal(bits(run_gpu(w, num_units=0)), bits(outs[0]))
    assert torch.equal(bits(run_gpu(w, num_units=7)), bits(outs[7]))


# Balancing chunks: the last part of every unit's tile range is cut into
# chunks that the first warps to run out of work claim at run time.  The
# workloads here give each unit enough tiles (few units) for the chunks to be
# used.
BALANCE = [(64, 3, 0), (64, 4, 500), (64, 1, 999), (200, 2, 0), (37, 0, 0), (150, 3, 700)]


@pytest.mark.parametrize("units,balance,permille", BALANCE, ids=[f"u{u}-c{c}-s{s}" for u, c, s in BALANCE])
def test_balancing_chunks_match_oracle_and_repeat_bitwise(units, balance, permille):
    w = W.uniform_gqa(batch=10, len_lo=100, len_hi=3000, seed=13)
    ref, _, _ = oracle.workload_decode(w)
    ws = pkv.new_workspace(pkv.paged_attention_workspace_size(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim,
                                                              w.dtype, balance_chunks=balance))
    kw = dict(num_units=units, balance_chunks=balance, static_permille=permille, workspace=ws)
    out = run_gpu(w, **kw)
    assert_close(out, ref, w.dtype, what=str(kw))
    for _ in range(3):   # which warp runs a chunk varies; the bits do not
        assert torch.equal(bits(run_gpu(w, **kw)), bits(out))


@pytest.mark.parametrize("simt", [False, True])
def test_balancing_chunks_on_mha_and_simt_paths(simt):
    w = W.lognormal_mha(batch=24, seed=31)
    ref, _, _ = oracle.workload_decode(w)
    for units, balance in ((48, 4), (48, 0)):
        out = run_gpu(w, num_units=units, balance_chunks=balance, force_simt=simt)
        assert_close(out, ref, w.dtype, what=f"mha units={units} balance={balance} simt={simt}")


def test_workspace_not_cleared_is_flagged_then_reset():
    w = W.uniform_gqa(batch=10, len_lo=100, len_hi=3000, seed=13)
    ref, _, _ = oracle.workload_decode(w)
    need = pkv.paged_attention_workspace_size(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.dtype,
                                              balance_chunks=3)
    for fill in (0x7F, 0xFF):   # a large positive and a negative claim counter
        ws = torch.full((need,), fill, dtype=torch.uint8, device="cuda")
        run_gpu(w, num_units=64, workspace=ws, check_errors=False, balance_chunks=3)
        assert pkv.pkv_get_device_error() & pkv.DEVERR_SCHEDULE
        out = run_gpu(w, num_units=64, workspace=ws, balance_chunks=3)   # the launch left the counter at zero
        assert_close(out, ref, w.dtype, what=f"after fill {fill:#x}")


def test_one_unit_no_split_matches_oracle_on_every_path():
    for simt in (False, True):
        w = W.build_workload("one", [3, 40, 517], 8, 2, 128, torch.bfloat16, seed=14)
        out = run_gpu(w, num_units=1, force_simt=simt)
        ref, _, _ = oracle.workload_decode(w)
        assert_close(out, ref, w.dtype, what=f"one unit simt={simt}")


def _moved(w, perm):
    """The same workload with physical block p moved to perm[p] (tables and
    slots rewritten to match)."""
    m = W.uniform_gqa(batch=8, len_lo=30, len_hi=1200, seed=15)
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(w.num_blocks)
    m.k_cache, m.v_cache = w.k_cache[inv].clone(), w.v_cache[inv].clone()
    bt = w.block_tables.clone()
    bt[bt >= 0] = perm[bt[bt >= 0].long()].to(torch.int32)
    m.block_tables = bt
    m.slot_mapping = perm[w.slot_mapping // 16] * 16 + w.slot_mapping % 16
    return m


def test_block_placement_does_not_change_a_bit():
    a = W.uniform_gqa(batch=8, len_lo=30, len_hi=1200, seed=15)
    shuffled = _moved(a, torch.randperm(a.num_blocks, generator=torch.Generator().manual_seed(77)))
    # Contiguous placement: the blocks of sequence 0, then sequence 1, ... in
    # logical order (the layout of a non-paged, slab cache).
    order = []
    for b, n in enumerate(a.lens()):
        order += a.block_tables[b, : (n + 15) // 16].tolist()
    rest = [p for p in range(a.num_blocks) if p not in set(order)]
    perm = torch.empty(a.num_blocks, dtype=torch.long)
    perm[torch.tensor(order + rest)] = torch.arange(a.num_blocks)
    contiguous = _moved(a, perm)
    assert (contiguous.block_tables[0, 1:4] - contiguous.block_tables[0, :3] == 1).all()
    oa, ob, oc = run_gpu(a), run_gpu(shuffled), run_gpu(contiguous)
    assert torch.equal(bits(oa), bits(ob))
    assert torch.equal(bits(oa), bits(oc))   # paged == contiguous placement


def test_shared_prefix_equals_private_copies():
    lens = [512 + 40, 512 + 100, 512 + 17, 512 + 256]
    s = W.build_workload("sh", lens, 16, 2, 128, torch.bfloat16, seed=16, groups=[([0, 1, 2, 3], 512)])
    out_shared = run_gpu(s)
    pb = s.block_tables[0, :32].tolist()
    extra = 4 * 32
    kc = torch.cat([s.k_cache, torch.zeros((extra,) + s.k_cache.shape[1:], dtype=s.k_cache.dtype)])
    vc = torch.cat([s.v_cache, torch.zeros((extra,) + s.v_cache.shape[1:], dtype=s.v_cache.dtype)])
    bt = s.block_tables.clone()
    nxt = s.num_blocks
    for b in range(4):
        for j, p in enumerate(pb):
            kc[nxt], vc[nxt], bt[b, j] = s.k_cache[p], s.v_cache[p], nxt
            nxt += 1
    s.k_cache, s.v_cache, s.block_tables = kc, vc, bt
    assert torch.equal(bits(run_gpu(s)), bits(out_shared))


def test_gqa_equals_repeated_mha_on_gpu():
    w = W.build_workload("gqa", [40, 300], 8, 2, 128, torch.float16, seed=17)
    m = W.build_workload("gqa", [40, 300], 8, 2, 128, torch.float16, seed=17)
    m.k_cache = w.k_cache.repeat_interleave(4, dim=1).contiguous()
    m.v_cache = w.v_cache.repeat_interleave(4, dim=1).contiguous()
    m.k_new = w.k_new.repeat_interleave(4, dim=1).contiguous()
    m.v_new = w.v_new.repeat_interleave(4, dim=1).contiguous()
    m.n_kv_heads = 8
    ref, _, _ = oracle.workload_decode(w)
    assert_close(run_gpu(w), ref, w.dtype, what="gqa")
    assert_close(run_gpu(m), ref, w.dtype, what="repeated mha")


def test_context_one_returns_v():
    w = W.build_workload("ctx1", [1] * 9, 32, 8, 128, torch.bfloat16, seed=18)
    out = run_gpu(w)
    G = 4
    for b in range(9):
        for h in range(32):
            assert torch.equal(bits(out[b, h]), bits(w.v_new[b, h // G]))


def test_scale_zero_gives_mean_of_v():
    w = W.build_workload("s0", [7, 64, 129], 8, 2, 64, torch.float32, seed=19, scale=0.0, append=False)
    ref, _, _ = oracle.workload_decode(w)
    assert_close(run_gpu(w), ref, w.dtype, what="scale 0")


def test_deterministic():
    w = W.lognormal_mha(batch=32, seed=20)
    assert torch.equal(bits(run_gpu(w)), bits(run_gpu(w)))


# --- edge cases ---

def test_empty_and_boundary_contexts():
    lens = [0, 1, 15, 16, 17, 0, 48, 64]
    w = W.build_workload("edge", [max(1, n) for n in lens], 8, 2, 128, torch.bfloat16, seed=21,
                         append=False, max_blocks_per_seq=4)
    w.context_lens = torch.tensor(lens, dtype=torch.int32)   # 64 = max_blocks * 16 exactly
    out = run_gpu(w)
    ref, _, _ = oracle.workload_decode(w)
    assert torch.equal(out[0], torch.zeros_like(out[0])) and torch.equal(out[5], torch.zeros_like(out[5]))
    assert_close(out, ref, w.dtype, what="edge")


def test_all_sequences_empty():
    w = W.build_workload("allempty", [1, 1, 1], 4, 4, 64, torch.float16, seed=22, append=False)
    w.context_lens = torch.zeros(3, dtype=torch.int32)
    out = run_gpu(w)
    assert torch.equal(out, torch.zeros_like(out))


def test_empty_batch_is_a_no_op():
    dev = torch.device("cuda")
    q = torch.zeros(0, 8, 128, dtype=torch.bfloat16, device=dev)
    cache = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16, device=dev)
    out = pkv.paged_attention_decode(q, cache, cache, torch.zeros(0, 1, dtype=torch.int32, device=dev),
                                     torch.zeros(0, dtype=torch.int32, device=dev), 0.1)
    assert out.shape == (0, 8, 128)


def test_maximum_batch():
    g = torch.Generator().manual_seed(23)
    lens = torch.randint(1, 40, (4096,), generator=g).tolist()
    w = W.build_workload("maxbatch", lens, 4, 1, 64, torch.bfloat16, seed=23)
    check_workload(w, rows=sample_rows(w, 200))


def test_explicit_workspace_and_too_small_workspace():
    w = W.uniform_gqa(batch=8, len_lo=500, len_hi=3000, seed=24)
    need = pkv.paged_attention_workspace_size(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.dtype)
    ws = pkv.new_workspace(need)
    a = run_gpu(w, workspace=ws)
    b = run_gpu(w)
    assert torch.equal(bits(a), bits(b))
    with pytest.raises(pkv.PagedKVError) as e:
        run_gpu(w, workspace=torch.empty(need - 256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 5


# --- device-side range checks (no trap; a flag and a defined result) ---

# A block table entry outside the pool: nothing is read from it, its tokens
# are left out of the softmax (a row left with no token is a zero row), and
# the flag is set.  The oracle of the same workload without those blocks
# gives the expected result.
@pytest.mark.parametrize("simt,units", [(False, 0), (False, 7), (True, 0), (True, 7)])
def test_bad_block_id_is_left_out_and_flagged(simt, units):
    w = W.build_workload("badblk", [40, 300, 200, 20, 129], 8, 2, 128, torch.bfloat16, seed=25, append=False)
    bad = {0: [1], 1: [3, 7, 18], 2: [0], 3: [0, 1], 4: [8]}   # middle, first, every and last (partial) blocks
    ref, _, _ = oracle.workload_decode(drop_blocks(w, bad))
    for b, js in bad.items():
        for i, j in enumerate(js):
            w.block_tables[b, j] = w.num_blocks + 5 if i % 2 == 0 else -3
    out = run_gpu(w, check_errors=False, force_simt=simt, num_units=units)
    assert pkv.pkv_get_device_error() & pkv.DEVERR_BLOCK_ID
    assert pkv.pkv_get_device_error() == 0   # read clears
    assert torch.equal(out[3], torch.zeros_like(out[3]))   # every block bad: a zero row
    assert_close(out, ref, w.dtype, what=f"bad block ids simt={simt} units={units}")


# The failure path of the bounded waits: unit 3's copies are never issued, so
# its consumer's wait (10 ms here) runs out.  The launch must return with the
# timeout bit set (every thread reaches the grid barrier), and the next call
# with default settings must be clean and right.
@pytest.mark.parametrize("simt", [False, True])
def test_bounded_wait_runs_out_and_the_next_call_is_clean(simt):
    w = W.uniform_gqa(batch=8, len_lo=200, len_hi=2000, seed=27)
    ref, _, _ = oracle.workload_decode(w)
    run_gpu(w, check_errors=False, force_simt=simt, wait_limit_us=10000, test_withhold_unit=3)
    assert pkv.pkv_get_device_error() & pkv.DEVERR_TIMEOUT
    out = run_gpu(w, force_simt=simt)
    assert_close(out, ref, w.dtype, what=f"after a timed-out launch, simt={simt}")


def test_withhold_hook_rejects_negative_values():
    w = W.build_workload("neg", [20], 4, 4, 64, torch.bfloat16, seed=28, append=False)
    with pytest.raises(pkv.PagedKVError) as e:
        run_gpu(w, wait_limit_us=-1)
    assert e.value.status == 1


def test_context_beyond_table_sets_flag():
    w = W.build_workload("badctx", [20, 20], 4, 4, 64, torch.bfloat16, seed=26, append=False,
                         max_blocks_per_seq=2)
    w.context_lens = torch.tensor([20, 33], dtype=torch.int32)   # table covers 32 tokens
    run_gpu(w, check_errors=False)
    assert pkv.pkv_get_device_error() & pkv.DEVERR_CONTEXT


def test_tensor_map_cache_follows_reused_addresses_and_shapes():
    # Encoded tensor maps are cached per (address, dtype, shape).  A cache
    # freed and replaced by another at the same address -- with another
    # shape, or the same shape and other contents -- must still decode right.
    dev = torch.device("cuda")
    for seed, nb_extra in ((71, 0), (72, 37), (73, 37)):
        w = W.build_workload("mapcache", [40, 300, 129], 8, 2, 128, torch.bfloat16, seed=seed,
                             pool_blocks=60 + nb_extra)
        ref, _, _ = oracle.workload_decode(w)
        out = run_gpu(w)
        assert_close(out, ref, w.dtype, what=f"seed {seed} pool {w.num_blocks}")
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
