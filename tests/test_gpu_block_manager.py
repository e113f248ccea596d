"""Copy-on-write block copies on the GPU (paged_kv_copy_blocks) bit for bit
against plain indexing on the CPU, and a serving-style run in which the C++
block manager drives forks, prefix-cache hits, appends, copies and decodes
on the GPU while the CPU oracle replays the same host decisions on its own
copy of the cache."""

import random

import pytest
import torch

import oracle
import oracle.block_manager as model
import paged_kv_cache_386_b200 as pkv
from tests.gpu_helpers import assert_close, bits

pytestmark = pytest.mark.gpu


def _cache(num_blocks, n_kv, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn((num_blocks, n_kv, 16, d), generator=g).to(dtype)
    v = torch.randn((num_blocks, n_kv, 16, d), generator=g).to(dtype)
    return k, v


def _pairs(num_blocks, n, seed):
    rng = random.Random(seed)
    ids = rng.sample(range(num_blocks), 2 * n)
    return ids[:n], ids[n:]          # dst disjoint from src and from itself


@pytest.mark.parametrize("dtype,n_kv,d,num_blocks,n_pairs", [
    (torch.bfloat16, 8, 128, 300, 37),
    (torch.float16, 1, 64, 50, 1),
    (torch.float32, 4, 128, 64, 20),
    (torch.bfloat16, 8, 128, 12000, 4096),
])
def test_copy_blocks_bit_exact(dtype, n_kv, d, num_blocks, n_pairs):
    k, v = _cache(num_blocks, n_kv, d, dtype, seed=n_pairs)
    k.view(-1)[::97] = float("nan")   # canaries: copied as bits
    src, dst = _pairs(num_blocks, n_pairs, seed=num_blocks)
    kd, vd = k.cuda(), v.cuda()
    pkv.paged_kv_copy_blocks(kd, vd, torch.tensor(src, dtype=torch.int32).cuda(),
                             torch.tensor(dst, dtype=torch.int32).cuda())
    assert pkv.pkv_get_device_error() == 0
    ek, ev = k.clone(), v.clone()
    ek[dst], ev[dst] = k[src], v[src]
    assert torch.equal(bits(kd.cpu()), bits(ek)) and torch.equal(bits(vd.cpu()), bits(ev))


def test_copy_blocks_bad_id_skips_pair_and_sets_flag():
    k, v = _cache(16, 2, 64, torch.bfloat16, seed=3)
    kd, vd = k.cuda(), v.cuda()
    src = torch.tensor([1, 16, 2], dtype=torch.int32).cuda()
    dst = torch.tensor([5, 6, -1], dtype=torch.int32).cuda()
    pkv.paged_kv_copy_blocks(kd, vd, src, dst)
    assert pkv.pkv_get_device_error() & pkv.DEVERR_BLOCK_ID
    ek, ev = k.clone(), v.clone()
    ek[5], ev[5] = k[1], v[1]
    assert torch.equal(bits(kd.cpu()), bits(ek)) and torch.equal(bits(vd.cpu()), bits(ev))


def _serve(seed, dtype, n_q, n_kv, d, num_blocks, steps):
    """Prompts (some sharing a system prompt through the prefix cache), forks
    for parallel samples, then decode steps; each step appends one token per
    live sequence, copies the copy-on-write blocks, and decodes."""
    rng = random.Random(seed)
    g = torch.Generator().manual_seed(seed)
    bs = 16
    k_cpu, v_cpu = _cache(num_blocks, n_kv, d, dtype, seed)
    k_gpu, v_gpu = k_cpu.cuda(), v_cpu.cuda()
    bm = pkv.BlockManager(num_blocks, bs, prefix_cache=True)
    system = [rng.randrange(30000) for _ in range(16 * 6)]
    live, next_id = [], 0
    for p in range(6):
        prompt = system[:rng.choice([0, 32, 96])] + [rng.randrange(30000) for _ in range(rng.randrange(1, 60))]
        cached = bm.add_sequence(next_id, len(prompt), pkv.pkv_bm_hash_blocks(prompt, bs))
        # Prefill of the non-cached part: the prompt's K/V enter through append.
        bt, _ = bm.tables([next_id], num_blocks)
        slots = torch.tensor([int(bt[0, j // bs]) * bs + j % bs for j in range(cached, len(prompt))],
                             dtype=torch.int64)
        kn = torch.randn((slots.numel(), n_kv, d), generator=g).to(dtype)
        vn = torch.randn((slots.numel(), n_kv, d), generator=g).to(dtype)
        if slots.numel():
            pkv.paged_kv_append(kn.cuda(), vn.cuda(), slots.cuda(), k_gpu, v_gpu)
            oracle.kv_append(kn, vn, slots, k_cpu, v_cpu, bs)
        live.append(next_id)
        next_id += 1
        if p % 2 == 0:                       # parallel samples of this prompt
            for _ in range(rng.randint(1, 3)):
                bm.fork(live[-1], next_id)
                live.append(next_id)
                next_id += 1
    worst = {}
    copies_seen = 0
    for step in range(steps):
        slots, src, dst = bm.append(live)
        copies_seen += src.numel()
        if src.numel():
            pkv.paged_kv_copy_blocks(k_gpu, v_gpu, src.cuda(), dst.cuda())
            k_cpu[dst.long()], v_cpu[dst.long()] = k_cpu[src.long()], v_cpu[src.long()]
        kn = torch.randn((len(live), n_kv, d), generator=g).to(dtype)
        vn = torch.randn((len(live), n_kv, d), generator=g).to(dtype)
        pkv.paged_kv_append(kn.cuda(), vn.cuda(), slots.cuda(), k_gpu, v_gpu)
        oracle.kv_append(kn, vn, slots, k_cpu, v_cpu, bs)
        bt, cl = bm.tables(live, num_blocks)
        bt = bt[:, :int((bt != -1).sum(1).max())].contiguous()
        q = torch.randn((len(live), n_q, d), generator=g).to(dtype)
        scale = d ** -0.5
        out = pkv.paged_attention_decode(q.cuda(), k_gpu, v_gpu, bt.cuda(), cl.cuda(), scale).cpu()
        assert pkv.pkv_get_device_error() == 0
        ref = oracle.paged_decode(q, k_cpu, v_cpu, bt, cl, scale)
        worst = assert_close(out, ref, dtype, what=f"step {step}")
        if step % 5 == 4 and len(live) > 2:   # a sequence finishes
            bm.free(live.pop(rng.randrange(len(live))))
    assert torch.equal(bits(k_gpu.cpu()), bits(k_cpu)) and torch.equal(bits(v_gpu.cpu()), bits(v_cpu))
    assert copies_seen > 0
    bm.close()
    return worst


@pytest.mark.parametrize("dtype,n_q,n_kv,d", [(torch.bfloat16, 32, 8, 128), (torch.float16, 8, 8, 64)])
def test_block_manager_drives_decode(dtype, n_q, n_kv, d):
    _serve(seed=7, dtype=dtype, n_q=n_q, n_kv=n_kv, d=d, num_blocks=400, steps=20)
