"""CPU oracle for paged KV append and paged decode attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It is independent of the CUDA
library: it shares no code, header or helper with it, and neither imports
the other.

* :func:`kv_append` / :func:`paged_decode` call the plain C fp64 oracle in
  ``pkv_oracle.c`` (built into ``liboracle.so`` by :func:`build`).
* :mod:`oracle.brute` is a second, pure-Python implementation in
  high-precision decimal arithmetic for tiny cases.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np
import torch

HERE = Path(__file__).resolve().parent
SRC = HERE / "pkv_oracle.c"
LIB = HERE / "liboracle.so"

ORC_DTYPE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
ERRORS = {-1: "invalid argument", -2: "slot beyond pool", -3: "block id out of range",
          -4: "context length out of range", -5: "out of memory"}


class OracleError(RuntimeError):
    pass


def build(src: Path = SRC, out: Path = LIB, extra: tuple[str, ...] = ()) -> Path:
    """Compile the C oracle with gcc (IEEE semantics: no fast-math)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-Wall", "-Wextra",
           *extra, "-o", str(out), str(src), "-lm"]
    subprocess.run(cmd, check=True)
    return out


_lib = None


def load(path: Path | None = None) -> ctypes.CDLL:
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(str(path)))
    if _lib is None:
        if not LIB.exists() or LIB.stat().st_mtime < SRC.stat().st_mtime:
            build()
        _lib = _bind(ctypes.CDLL(str(LIB)))
    return _lib


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    p, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.oracle_kv_append.argtypes = [p, p, p, i32, p, p, i32, i32, i32, i32, i32]
    lib.oracle_kv_append.restype = ctypes.c_int
    lib.oracle_paged_decode.argtypes = [p, p, p, i32, p, i32, p, i32, i32, ctypes.c_double,
                                        i32, i32, i32, i32, p, p, i32, i32]
    lib.oracle_paged_decode.restype = ctypes.c_int
    lib.oracle_widen.argtypes = [p, i32, i64, p]
    lib.oracle_widen.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_paged_decode_mq.argtypes = [p, p, p, i32, p, i32, p, i32, i32, ctypes.c_double, i32, i32, i32, i32,
                                           i32, p, i32]
    lib.oracle_paged_decode_mq.restype = ctypes.c_int
    lib.oracle_kv_append_int8.argtypes = [p, p, i32, p, i32, p, i32, i32, i32, i32]
    lib.oracle_kv_append_int8.restype = ctypes.c_int
    lib.oracle_paged_decode_int8.argtypes = [p, i32, p, p, i32, p, i32, i32, ctypes.c_double, i32, i32, i32, i32,
                                             p, p, i32, i32]
    lib.oracle_paged_decode_int8.restype = ctypes.c_int
    return lib


def _ptr(t: torch.Tensor) -> int:
    assert t.device.type == "cpu" and t.is_contiguous()
    return t.data_ptr()


def _check(rc: int) -> None:
    if rc != 0:
        raise OracleError(ERRORS.get(rc, f"oracle error {rc}"))


def kv_append(k, v, slot_mapping, k_cache, v_cache, block_size: int, lib=None) -> None:
    """In-place append of ``k``/``v`` ``[tokens, n_kv, d]`` into CPU caches."""
    lib = lib or load()
    num_blocks, n_kv, bs, d = k_cache.shape
    assert bs == block_size
    k, v = k.contiguous(), v.contiguous()
    sm = slot_mapping.to(torch.int64).contiguous()
    _check(lib.oracle_kv_append(_ptr(k), _ptr(v), _ptr(sm), k.shape[0], _ptr(k_cache),
                                _ptr(v_cache), num_blocks, bs, n_kv, d, ORC_DTYPE[k.dtype]))


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                 rows=None, n_threads: int = 0, lib=None) -> torch.Tensor:
    """fp64 ``[batch, n_q, d]`` attention output.  ``rows`` optionally limits
    the work to a list of (b, h) pairs; other rows are returned as NaN."""
    lib = lib or load()
    B, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_cache.shape
    assert d2 == d and k_cache.dtype == q.dtype == v_cache.dtype
    q = q.contiguous()
    bt = block_tables.to(torch.int32).contiguous()
    cl = context_lens.to(torch.int32).contiguous()
    out = torch.full((B, n_q, d), float("nan"), dtype=torch.float64)
    if rows is not None:
        r = torch.as_tensor(rows, dtype=torch.int32).reshape(-1, 2).contiguous()
        rp, nr = _ptr(r), r.shape[0]
    else:
        rp, nr = None, 0
    _check(lib.oracle_paged_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), ORC_DTYPE[q.dtype],
                                   _ptr(bt), bt.shape[1], _ptr(cl), B, num_blocks, float(scale),
                                   n_q, n_kv, d, bs, _ptr(out), rp, nr, int(n_threads)))
    return out


def widen(t: torch.Tensor, lib=None) -> np.ndarray:
    """Exact widening of an f32/f16/bf16 CPU tensor to float64, by the oracle's
    own conversion routines."""
    lib = lib or load()
    t = t.contiguous()
    out = np.empty(t.numel(), dtype=np.float64)
    _check(lib.oracle_widen(_ptr(t), ORC_DTYPE[t.dtype], t.numel(), out.ctypes.data))
    return out.reshape(tuple(t.shape))


def max_threads(lib=None) -> int:
    return int((lib or load()).oracle_max_threads())


def workload_decode(w, rows=None, n_threads: int = 0, lib=None):
    """Oracle result for a workload after its append step: returns
    ``(out_fp64, k_cache_after, v_cache_after)``."""
    kc, vc = w.k_cache.clone(), w.v_cache.clone()
    if w.appended:
        kv_append(w.k_new, w.v_new, w.slot_mapping, kc, vc, w.block_size, lib=lib)
    out = paged_decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, rows=rows,
                       n_threads=n_threads, lib=lib)
    return out, kc, vc


def paged_decode_mq(q, k_cache, v_cache, block_tables, context_lens, scale: float, n_threads: int = 0,
                    lib=None) -> torch.Tensor:
    """fp64 ``[batch, q_len, n_q, d]`` multi-query attention: query i of a
    sequence sees its context up to position ``ctx - q_len + i``."""
    lib = lib or load()
    B, q_len, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_cache.shape
    assert d2 == d and k_cache.dtype == q.dtype == v_cache.dtype
    q = q.contiguous()
    bt = block_tables.to(torch.int32).contiguous()
    cl = context_lens.to(torch.int32).contiguous()
    out = torch.full((B, q_len, n_q, d), float("nan"), dtype=torch.float64)
    _check(lib.oracle_paged_decode_mq(_ptr(q), _ptr(k_cache), _ptr(v_cache), ORC_DTYPE[q.dtype], _ptr(bt),
                                      bt.shape[1], _ptr(cl), B, num_blocks, float(scale), n_q, n_kv, d, bs, q_len,
                                      _ptr(out), int(n_threads)))
    return out


def workload_decode_mq(w, n_threads: int = 0, lib=None):
    """Oracle for a multi-query workload: append its q_len new tokens per
    sequence, then the causal multi-query decode.  Returns
    ``(out_fp64 [B, q_len, n_q, d], k_cache_after, v_cache_after)``."""
    kc, vc = w.k_cache.clone(), w.v_cache.clone()
    if w.appended:
        kv_append(w.k_new, w.v_new, w.slot_mapping, kc, vc, w.block_size, lib=lib)
    q = w.q if w.q.dim() == 4 else w.q.unsqueeze(1)
    out = paged_decode_mq(q, kc, vc, w.block_tables, w.context_lens, w.scale, n_threads=n_threads, lib=lib)
    return out, kc, vc


def kv_append_int8(k, v, slot_mapping, cache, lib=None) -> None:
    """In-place quantising append into the INT8 cache, a CPU uint8 tensor
    ``[blocks, n_kv, 32 * d + 128]`` of records (layout in pkv_oracle.c)."""
    lib = lib or load()
    num_blocks, n_kv, rb = cache.shape
    d = k.shape[-1]
    assert rb == 32 * d + 128 and cache.dtype == torch.uint8
    k, v = k.contiguous(), v.contiguous()
    sm = slot_mapping.to(torch.int64).contiguous()
    _check(lib.oracle_kv_append_int8(_ptr(k), _ptr(v), ORC_DTYPE[k.dtype], _ptr(sm), k.shape[0], _ptr(cache),
                                     num_blocks, 16, n_kv, d))


def paged_decode_int8(q, cache, block_tables, context_lens, scale: float, rows=None, n_threads: int = 0,
                      lib=None) -> torch.Tensor:
    """fp64 ``[batch, n_q, d]`` attention over the dequantised INT8 cache."""
    lib = lib or load()
    B, n_q, d = q.shape
    num_blocks, n_kv, rb = cache.shape
    assert rb == 32 * d + 128
    q = q.contiguous()
    bt = block_tables.to(torch.int32).contiguous()
    cl = context_lens.to(torch.int32).contiguous()
    out = torch.full((B, n_q, d), float("nan"), dtype=torch.float64)
    r = None
    n_rows = 0
    if rows is not None:
        r = torch.as_tensor(rows, dtype=torch.int32).reshape(-1, 2).contiguous()
        n_rows = r.shape[0]
    _check(lib.oracle_paged_decode_int8(_ptr(q), ORC_DTYPE[q.dtype], _ptr(cache), _ptr(bt), bt.shape[1], _ptr(cl),
                                        B, num_blocks, float(scale), n_q, n_kv, d, 16, _ptr(out),
                                        _ptr(r) if r is not None else None, n_rows, n_threads))
    return out


def workload_decode_int8(w, rows=None, n_threads: int = 0, lib=None):
    """Oracle for a workload held in the INT8 cache: every cached token and
    the appended one go through the quantising append, then the decode runs
    over the dequantised cache.  Returns ``(out_fp64, cache)``."""
    import workloads as W
    cache = W.int8_cache_buffers(w)
    kr, vr, slots = W.cached_token_rows(w)
    kv_append_int8(kr, vr, slots, cache, lib=lib)
    if w.appended:
        kv_append_int8(w.k_new, w.v_new, w.slot_mapping, cache, lib=lib)
    out = paged_decode_int8(w.q, cache, w.block_tables, w.context_lens, w.scale, rows=rows, n_threads=n_threads,
                            lib=lib)
    return out, cache


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
