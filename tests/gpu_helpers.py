"""Shared helpers of the GPU parity tests: run a workload through the C-ABI
(append, then decode) and compare with the CPU oracle on the same seeded
inputs."""

from __future__ import annotations

import torch

import oracle
import paged_kv_cache_386_b200 as pkv

# Tolerances of the decode output against the fp64 oracle on the same rounded
# inputs: fp32 data max-abs 1e-5; 16-bit data (fp32 accumulation) max-abs
# 2e-2 and relative L2 error 5e-3.
TOL = {
    torch.float32: {"max_abs": 1e-5, "rel_l2": None},
    torch.float16: {"max_abs": 2e-2, "rel_l2": 5e-3},
    torch.bfloat16: {"max_abs": 2e-2, "rel_l2": 5e-3},
}


def bits(t: torch.Tensor) -> torch.Tensor:
    """Integer view for bit-exact comparisons (NaN canaries compare equal)."""
    return t.contiguous().view(torch.int32 if t.element_size() == 4 else torch.int16)


def run_gpu(w, num_units: int = 0, force_simt: bool = False, check_errors: bool = True,
            return_cache: bool = False, workspace=None, balance_chunks: int = 0, static_permille: int = 0,
            **hooks):
    dev = torch.device("cuda")
    kc, vc = w.k_cache.to(dev), w.v_cache.to(dev)
    if w.appended:
        pkv.paged_kv_append(w.k_new.to(dev), w.v_new.to(dev), w.slot_mapping.to(dev), kc, vc)
    out = pkv.paged_attention_decode(w.q.to(dev), kc, vc, w.block_tables.to(dev), w.context_lens.to(dev),
                                     w.scale, num_units=num_units, force_simt=force_simt,
                                     workspace=workspace, balance_chunks=balance_chunks,
                                     static_permille=static_permille, **hooks)
    torch.cuda.synchronize()
    if check_errors:
        assert pkv.pkv_get_device_error() == 0
    if return_cache:
        return out.cpu(), kc.cpu(), vc.cpu()
    return out.cpu()


def errors(out: torch.Tensor, ref: torch.Tensor, rows=None) -> dict:
    o = out.double()
    if rows is not None:
        idx = torch.as_tensor(rows, dtype=torch.long)
        o = o[idx[:, 0], idx[:, 1]]
        ref = ref[idx[:, 0], idx[:, 1]]
    diff = (o - ref)
    max_abs = diff.abs().max().item() if diff.numel() else 0.0
    denom = ref.norm().item()
    rel = diff.norm().item() / denom if denom > 0 else diff.norm().item()
    return {"max_abs": max_abs, "rel_l2": rel, "finite": bool(torch.isfinite(o).all())}


def assert_close(out: torch.Tensor, ref: torch.Tensor, dtype: torch.dtype, rows=None, what: str = ""):
    e = errors(out, ref, rows)
    tol = TOL[dtype]
    assert e["finite"], f"{what}: non-finite output"
    assert e["max_abs"] <= tol["max_abs"], f"{what}: max abs error {e['max_abs']:.3e} > {tol['max_abs']}"
    if tol["rel_l2"] is not None:
        assert e["rel_l2"] <= tol["rel_l2"], f"{what}: rel L2 error {e['rel_l2']:.3e} > {tol['rel_l2']}"
    return e


def sample_rows(w, n: int, seed: int = 0):
    """n (sequence, q head) pairs: the first and last of each, plus random ones."""
    g = torch.Generator().manual_seed(seed)
    rows = {(0, 0), (w.batch - 1, w.n_q_heads - 1)}
    while len(rows) < min(n, w.batch * w.n_q_heads):
        rows.add((int(torch.randint(w.batch, (1,), generator=g)), int(torch.randint(w.n_q_heads, (1,), generator=g))))
    return sorted(rows)


def check_workload(w, rows=None, **kw):
    """GPU append + decode vs the oracle; the append is checked bit for bit."""
    out, kc, vc = run_gpu(w, return_cache=True, **kw)
    ref, okc, ovc = oracle.workload_decode(w, rows=rows)
    assert torch.equal(bits(kc), bits(okc)) and torch.equal(bits(vc), bits(ovc)), "append not bit-exact"
    return assert_close(out, ref, w.dtype, rows=rows, what=w.name)


def drop_blocks(w, drop: dict, **overrides):
    """The same workload with logical blocks ``drop[b]`` (a list of block
    indices) removed from sequence b's table and context: attention over the
    remaining keys.  The expected result of a decode whose table names those
    blocks with out-of-range ids (their tokens are left out)."""
    import copy
    m = copy.copy(w)
    bt = w.block_tables.clone()
    cl = w.context_lens.clone()
    for b, js in drop.items():
        n = int(cl[b])
        keep = [j for j in range((n + 15) // 16) if j not in set(js)]
        removed = sum(min(16, n - 16 * j) for j in js)
        row = torch.full((bt.shape[1],), -1, dtype=torch.int32)
        row[: len(keep)] = w.block_tables[b, keep]
        bt[b] = row
        cl[b] = n - removed
    m.block_tables, m.context_lens = bt, cl
    for k, v in overrides.items():
        setattr(m, k, v)
    return m
