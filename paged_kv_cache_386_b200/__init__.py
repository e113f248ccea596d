"""Paged KV cache for B200 (sm_100a): a thin Python binding of libpagedkv.so.

The functions below carry the names of the C entry points in
``include/pagedkv.h`` and only marshal arguments: every step of the append and
of the decode attention runs in the library's CUDA kernels.  There is no CPU
fallback: if the library is missing or no GPU is present the calls raise.

Tensors are torch CUDA tensors in the library's layout:

* ``k_cache``, ``v_cache``: ``[num_blocks, n_kv_heads, 16, head_dim]``
* ``q``, ``out``: ``[batch, n_q_heads, head_dim]``
* ``block_tables``: int32 ``[batch, max_blocks_per_seq]``
* ``context_lens``: int32 ``[batch]``
* ``slot_mapping``: int64 ``[num_tokens]``; ``k``, ``v``: ``[num_tokens, n_kv_heads, head_dim]``
"""

from __future__ import annotations

import ctypes
from pathlib import Path

import torch

__all__ = [
    "paged_kv_append", "paged_attention_decode", "paged_kv_append_and_decode", "paged_attention_decode_noalloc",
    "paged_attention_decode_cascade", "paged_attention_cascade_workspace_size",
    "paged_attention_workspace_size", "paged_kv_copy_blocks", "BlockManager", "pkv_bm_hash_blocks",
    "paged_kv_append_int8", "paged_attention_decode_int8", "int8_cache",
    "paged_attention_decode_mq", "paged_attention_mq_workspace_size",
    "pkv_get_device_error", "pkv_status_string", "pkv_version", "PagedKVError", "library_path",
    "DEVERR_BLOCK_ID", "DEVERR_CONTEXT", "DEVERR_SLOT", "DEVERR_TIMEOUT", "DEVERR_SCHEDULE", "new_workspace",
]

_LIB_PATH = Path(__file__).resolve().parent / "libpagedkv.so"

PKV_F32, PKV_F16, PKV_BF16 = 0, 1, 2
_DTYPE = {torch.float32: PKV_F32, torch.float16: PKV_F16, torch.bfloat16: PKV_BF16}

PKV_OK = 0
PKV_ERR_INVALID_ARG, PKV_ERR_NO_BLOCKS = 1, 6
DEVERR_BLOCK_ID, DEVERR_CONTEXT, DEVERR_SLOT, DEVERR_TIMEOUT, DEVERR_SCHEDULE = 0x1, 0x2, 0x4, 0x8, 0x10


class PagedKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {pkv_status_string(status)} (status {status})")


class _Options(ctypes.Structure):
    _fields_ = [("num_units", ctypes.c_int32), ("force_simt", ctypes.c_int32),
                ("balance_chunks", ctypes.c_int32), ("static_permille", ctypes.c_int32),
                ("wait_limit_us", ctypes.c_int32), ("test_withhold_unit", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 2)]


class _CascadeOptions(ctypes.Structure):
    _fields_ = [("prefix_splits", ctypes.c_int32), ("prefix_kernel", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 6)]


class _BMStats(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("free_blocks", ctypes.c_int32),
                ("cached_idle_blocks", ctypes.c_int32), ("used_blocks", ctypes.c_int32),
                ("cached_blocks", ctypes.c_int32), ("sequences", ctypes.c_int32),
                ("tokens", ctypes.c_int64), ("allocated_slots", ctypes.c_int64)]


_lib = None


def library_path() -> Path:
    return _LIB_PATH


def _load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not _LIB_PATH.exists():
        raise RuntimeError(f"CUDA library {_LIB_PATH} is not built: run "
                           "`python -m paged_kv_cache_386_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(str(_LIB_PATH))
    p, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    lib.paged_kv_append.argtypes = [p, p, p, i32, p, p, i32, i32, i32, i32, ctypes.c_int, p]
    lib.paged_kv_append.restype = ctypes.c_int
    lib.paged_attention_workspace_size.argtypes = [i32, i32, i32, i32, ctypes.c_int, ctypes.POINTER(sz)]
    lib.paged_attention_workspace_size.restype = ctypes.c_int
    lib.paged_attention_workspace_size_ex.argtypes = [i32, i32, i32, i32, ctypes.c_int, ctypes.POINTER(_Options),
                                                      ctypes.POINTER(sz)]
    lib.paged_attention_workspace_size_ex.restype = ctypes.c_int
    dec = [p, p, p, p, i32, p, i32, i32, f32, i32, i32, i32, i32, p, ctypes.c_int, p, sz, p]
    lib.paged_attention_decode.argtypes = dec
    lib.paged_attention_decode.restype = ctypes.c_int
    lib.paged_attention_decode_ex.argtypes = dec + [ctypes.POINTER(_Options)]
    lib.paged_attention_decode_ex.restype = ctypes.c_int
    lib.paged_kv_append_and_decode.argtypes = [p, p, p, p, i32, p, p, p, i32, p, i32, i32, f32, i32, i32, i32, i32,
                                               p, ctypes.c_int, p, sz, p]
    lib.paged_kv_append_and_decode.restype = ctypes.c_int
    lib.paged_attention_cascade_workspace_size.argtypes = [i32, i32, i32, i32, ctypes.c_int, ctypes.POINTER(sz)]
    lib.paged_attention_cascade_workspace_size.restype = ctypes.c_int
    lib.paged_attention_decode_cascade.argtypes = [p, p, p, i32, p, i32, p, p, p, i32, p, i32, i32, f32, i32, i32,
                                                   i32, i32, p, ctypes.c_int, p, sz, p]
    lib.paged_attention_decode_cascade.restype = ctypes.c_int
    lib.paged_attention_decode_cascade_ex.argtypes = lib.paged_attention_decode_cascade.argtypes + [
        ctypes.POINTER(_CascadeOptions)]
    lib.paged_attention_decode_cascade_ex.restype = ctypes.c_int
    lib.paged_attention_decode_noalloc.argtypes = dec[:15] + [p]
    lib.paged_attention_decode_noalloc.restype = ctypes.c_int
    lib.pkv_get_device_error.argtypes = [p, ctypes.POINTER(ctypes.c_uint32)]
    lib.pkv_get_device_error.restype = ctypes.c_int
    lib.pkv_status_string.argtypes = [ctypes.c_int]
    lib.pkv_status_string.restype = ctypes.c_char_p
    lib.pkv_version.argtypes = []
    lib.pkv_version.restype = ctypes.c_int32
    lib.paged_kv_copy_blocks.argtypes = [p, p, p, p, i32, i32, i32, i32, i32, ctypes.c_int, p]
    lib.paged_kv_copy_blocks.restype = ctypes.c_int
    lib.paged_attention_mq_workspace_size.argtypes = [i32, i32, i32, i32, i32, ctypes.c_int, ctypes.POINTER(sz)]
    lib.paged_attention_mq_workspace_size.restype = ctypes.c_int
    lib.paged_attention_decode_mq.argtypes = [p, p, p, p, i32, p, i32, i32, i32, f32, i32, i32, i32, i32, p,
                                              ctypes.c_int, p, sz, p]
    lib.paged_attention_decode_mq.restype = ctypes.c_int
    lib.paged_kv_append_int8.argtypes = [p, p, ctypes.c_int, p, i32, p, i32, i32, i32, i32, p]
    lib.paged_kv_append_int8.restype = ctypes.c_int
    lib.paged_attention_decode_int8.argtypes = [p, p, p, i32, p, i32, i32, f32, i32, i32, i32, i32, p,
                                                ctypes.c_int, p, sz, p]
    lib.paged_attention_decode_int8.restype = ctypes.c_int
    i64, u64 = ctypes.c_int64, ctypes.c_uint64
    for name, args in (("pkv_bm_create", [i32, i32, i32, ctypes.POINTER(p)]),
                       ("pkv_bm_hash_blocks", [p, i64, i32, u64, p]),
                       ("pkv_bm_add_sequence", [p, i64, i64, p, ctypes.POINTER(i64)]),
                       ("pkv_bm_fork", [p, i64, i64]),
                       ("pkv_bm_append", [p, p, i32, p, p, p, ctypes.POINTER(i32)]),
                       ("pkv_bm_free", [p, i64]),
                       ("pkv_bm_get_tables", [p, p, i32, i32, p, p]),
                       ("pkv_bm_stats", [p, ctypes.POINTER(_BMStats)]),
                       ("pkv_bm_refcount", [p, i32, ctypes.POINTER(i32)])):
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.pkv_bm_destroy.argtypes = [p]
    lib.pkv_bm_destroy.restype = None
    _lib = lib
    return lib


def _stream(stream, device=None) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _same_device(device, *tensors) -> None:
    for t in tensors:
        if t is not None and t.device != device:
            raise ValueError(f"every tensor must be on {device} (found {t.device})")


def _check_decode_io(q, k_cache, v_cache, out, *others) -> None:
    """The C layer sees raw pointers and q's dtype only: check here that the
    caches and out have q's dtype, that out has q's shape, and that every
    tensor is on q's device (the call runs with that device current)."""
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError(f"k_cache/v_cache dtype ({k_cache.dtype}, {v_cache.dtype}) must equal q's ({q.dtype})")
    if out.dtype != q.dtype or tuple(out.shape) != tuple(q.shape):
        raise ValueError(f"out must have q's dtype and shape ({q.dtype}, {tuple(q.shape)}), "
                         f"got ({out.dtype}, {tuple(out.shape)})")
    if not out.is_contiguous():
        raise ValueError("out must be contiguous")
    _same_device(q.device, k_cache, v_cache, out, *others)


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _check(status: int, where: str) -> None:
    if status != PKV_OK:
        raise PagedKVError(status, where)


def pkv_status_string(status: int) -> str:
    return _load().pkv_status_string(int(status)).decode()


def pkv_version() -> int:
    return int(_load().pkv_version())


def paged_kv_append(k, v, slot_mapping, k_cache, v_cache, block_size: int = 16, stream=None) -> None:
    """Write ``k[i]``, ``v[i]`` into slot ``slot_mapping[i]`` of the caches (in place)."""
    lib = _load()
    num_blocks, n_kv, bs, d = k_cache.shape
    if bs != block_size or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("cache shapes disagree")
    if (k.dtype != k_cache.dtype or v.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype
            or slot_mapping.dtype != torch.int64):
        raise ValueError("dtype mismatch (slot_mapping must be int64)")
    if tuple(k.shape[1:]) != (n_kv, d) or tuple(v.shape) != tuple(k.shape) or slot_mapping.shape[0] != k.shape[0]:
        raise ValueError("k, v must be [num_tokens, n_kv_heads, head_dim] and slot_mapping [num_tokens]")
    _same_device(k_cache.device, k, v, slot_mapping, v_cache)
    with torch.cuda.device(k_cache.device):
        _check(lib.paged_kv_append(_dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping"),
                                   k.shape[0], _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                   num_blocks, bs, n_kv, d, _DTYPE[k_cache.dtype], _stream(stream, k_cache.device)),
               "paged_kv_append")


def paged_attention_workspace_size(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                                   dtype: torch.dtype, balance_chunks: int = 0) -> int:
    out = ctypes.c_size_t(0)
    opts = _Options(balance_chunks=int(balance_chunks))
    _check(_load().paged_attention_workspace_size_ex(batch, n_q_heads, n_kv_heads, head_dim,
                                                     _DTYPE[dtype], ctypes.byref(opts), ctypes.byref(out)),
           "paged_attention_workspace_size")
    return int(out.value)


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A decode workspace: zero-filled device bytes, as the library requires
    before a workspace's first use (each call leaves it ready for the next)."""
    return torch.zeros(int(nbytes), dtype=torch.uint8, device=device or "cuda")


def paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, out=None,
                           workspace=None, num_units: int = 0, force_simt: bool = False,
                           balance_chunks: int = 0, static_permille: int = 0,
                           block_size: int = 16, stream=None, wait_limit_us: int = 0,
                           test_withhold_unit: int = -1):
    """Single-query attention through the block table; returns ``out``.
    With ``balance_chunks`` > 0 the workspace (see new_workspace) must be
    zero-filled before its first use.  ``wait_limit_us`` and
    ``test_withhold_unit`` are the failure-path test hooks of
    ``pkv_decode_options`` (a unit whose copies are never issued, so that its
    bounded wait runs out)."""
    lib = _load()
    B, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_cache.shape
    if d2 != d or bs != block_size or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if out is None:
        out = torch.empty_like(q)
    _check_decode_io(q, k_cache, v_cache, out, block_tables, context_lens, workspace)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    opts = _Options(num_units=int(num_units), force_simt=int(bool(force_simt)),
                    balance_chunks=int(balance_chunks), static_permille=int(static_permille),
                    wait_limit_us=int(wait_limit_us), test_withhold_unit=int(test_withhold_unit) + 1)
    with torch.cuda.device(q.device):
        _check(lib.paged_attention_decode_ex(
            _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
            _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"),
            B, num_blocks, float(scale), n_q, n_kv, d, bs, _dev(out, "out"), _DTYPE[q.dtype],
            ws_ptr, ws_bytes, _stream(stream, q.device), ctypes.byref(opts)), "paged_attention_decode")
    return out


def paged_kv_append_and_decode(q, k, v, slot_mapping, k_cache, v_cache, block_tables, context_lens, scale: float,
                               out=None, workspace=None, block_size: int = 16, stream=None):
    """paged_kv_append(k, v, slot_mapping, ...) then paged_attention_decode(q,
    ...) in one launch (the caches are written in place); returns ``out``."""
    lib = _load()
    B, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_cache.shape
    if d2 != d or bs != block_size or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if k.dtype != q.dtype or v.dtype != q.dtype or slot_mapping.dtype != torch.int64:
        raise ValueError("k and v must have q's dtype, slot_mapping int64")
    if tuple(k.shape[1:]) != (n_kv, d) or tuple(v.shape) != tuple(k.shape) or slot_mapping.shape[0] != k.shape[0]:
        raise ValueError("k, v must be [num_tokens, n_kv_heads, head_dim] and slot_mapping [num_tokens]")
    if out is None:
        out = torch.empty_like(q)
    _check_decode_io(q, k_cache, v_cache, out, k, v, slot_mapping, block_tables, context_lens, workspace)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    with torch.cuda.device(q.device):
        _check(lib.paged_kv_append_and_decode(
            _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping"), k.shape[0],
            _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(block_tables, "block_tables"),
            block_tables.shape[1], _dev(context_lens, "context_lens"), B, num_blocks, float(scale), n_q, n_kv, d,
            bs, _dev(out, "out"), _DTYPE[q.dtype], ws_ptr, ws_bytes, _stream(stream, q.device)),
            "paged_kv_append_and_decode")
    return out


def paged_attention_cascade_workspace_size(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                                           dtype: torch.dtype) -> int:
    out = ctypes.c_size_t(0)
    _check(_load().paged_attention_cascade_workspace_size(batch, n_q_heads, n_kv_heads, head_dim,
                                                          _DTYPE[dtype], ctypes.byref(out)),
           "paged_attention_cascade_workspace_size")
    return int(out.value)


def paged_attention_decode_cascade(q, k_cache, v_cache, prefix_block_tables, prefix_lens, seq_group,
                                   block_tables, context_lens, scale: float, out=None, workspace=None,
                                   block_size: int = 16, stream=None, prefix_splits: int = 0,
                                   prefix_kernel: int = 0):
    """Decode for sequences that share prefix blocks: group i's prefix
    (``prefix_lens[i]`` tokens in ``prefix_block_tables[i]``) is attended once
    per kv head for all its members (``seq_group[b] == i``), then each
    sequence's private suffix (``block_tables[b]``, ``context_lens[b]``
    tokens) continues from that state.  ``prefix_splits`` (1-4, 0 = default)
    and ``prefix_kernel`` (0 default, 1 tensor-memory, 2 mma.sync) are the
    tuning hooks of ``pkv_cascade_options``."""
    lib = _load()
    B, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_cache.shape
    if d2 != d or bs != block_size or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch")
    for t, name in ((prefix_block_tables, "prefix_block_tables"), (prefix_lens, "prefix_lens"),
                    (seq_group, "seq_group"), (block_tables, "block_tables"), (context_lens, "context_lens")):
        if t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")
    if out is None:
        out = torch.empty_like(q)
    _check_decode_io(q, k_cache, v_cache, out, prefix_block_tables, prefix_lens, seq_group, block_tables,
                     context_lens, workspace)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    n_groups = prefix_lens.shape[0]
    opts = _CascadeOptions(prefix_splits=int(prefix_splits), prefix_kernel=int(prefix_kernel))
    with torch.cuda.device(q.device):
        _check(lib.paged_attention_decode_cascade_ex(
            _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), n_groups,
            _dev(prefix_block_tables, "prefix_block_tables") if n_groups else None,
            prefix_block_tables.shape[1] if n_groups else 0,
            _dev(prefix_lens, "prefix_lens") if n_groups else None,
            _dev(seq_group, "seq_group") if n_groups else None,
            _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"),
            B, num_blocks, float(scale), n_q, n_kv, d, bs, _dev(out, "out"), _DTYPE[q.dtype],
            ws_ptr, ws_bytes, _stream(stream, q.device), ctypes.byref(opts)), "paged_attention_decode_cascade")
    return out


def paged_attention_decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, scale: float, out=None,
                                   block_size: int = 16, stream=None):
    """paged_attention_decode for callers that cannot allocate device memory:
    the split-context scratch is the library's static device array (shared by
    every call on the device, so calls must not overlap on the GPU)."""
    lib = _load()
    B, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_cache.shape
    if d2 != d or bs != block_size or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if out is None:
        out = torch.empty_like(q)
    _check_decode_io(q, k_cache, v_cache, out, block_tables, context_lens)
    with torch.cuda.device(q.device):
        _check(lib.paged_attention_decode_noalloc(
            _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
            _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"),
            B, num_blocks, float(scale), n_q, n_kv, d, bs, _dev(out, "out"), _DTYPE[q.dtype],
            _stream(stream, q.device)), "paged_attention_decode_noalloc")
    return out


def pkv_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error bits."""
    flags = ctypes.c_uint32(0)
    st = _load().pkv_get_device_error(_stream(stream), ctypes.byref(flags))
    if st not in (PKV_OK, 3):
        raise PagedKVError(st, "pkv_get_device_error")
    return int(flags.value)


def paged_kv_copy_blocks(k_cache, v_cache, src_blocks, dst_blocks, block_size: int = 16, stream=None) -> None:
    """Copy whole blocks ``src_blocks[p] -> dst_blocks[p]`` in both caches
    (the copy of copy-on-write)."""
    lib = _load()
    num_blocks, n_kv, bs, d = k_cache.shape
    if bs != block_size or tuple(v_cache.shape) != tuple(k_cache.shape) or v_cache.dtype != k_cache.dtype:
        raise ValueError("cache shapes disagree")
    if src_blocks.dtype != torch.int32 or dst_blocks.dtype != torch.int32 or src_blocks.shape != dst_blocks.shape:
        raise ValueError("src_blocks and dst_blocks must be int32 of one shape")
    n = src_blocks.numel()
    if n == 0:
        return
    _same_device(k_cache.device, v_cache, src_blocks, dst_blocks)
    with torch.cuda.device(k_cache.device):
        _check(lib.paged_kv_copy_blocks(_dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                        _dev(src_blocks, "src_blocks"), _dev(dst_blocks, "dst_blocks"), n,
                                        num_blocks, bs, n_kv, d, _DTYPE[k_cache.dtype],
                                        _stream(stream, k_cache.device)), "paged_kv_copy_blocks")


def _host(t: torch.Tensor, dtype: torch.dtype, name: str) -> torch.Tensor:
    t = torch.as_tensor(t, dtype=dtype)
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    return t.contiguous()


def pkv_bm_hash_blocks(tokens, block_size: int = 16, seed: int = 0) -> list[int]:
    """Chained FNV-1a keys of the full blocks of a prompt (host call)."""
    t = _host(tokens, torch.int32, "tokens").reshape(-1)
    n = t.numel() // block_size
    out = (ctypes.c_uint64 * max(n, 1))()
    _check(_load().pkv_bm_hash_blocks(t.data_ptr() if t.numel() else None, t.numel(), block_size,
                                      ctypes.c_uint64(seed & (2**64 - 1)), out), "pkv_bm_hash_blocks")
    return [int(out[i]) for i in range(n)]


class BlockManager:
    """Host block manager of the pool (C++ behind the pkv_bm_* entry points):
    free pool, per-sequence block tables, refcounted fork with copy-on-write
    of a shared last block, and an optional hash-keyed prefix cache with LRU
    eviction.  Everything runs on the host; the outputs feed
    paged_kv_copy_blocks, paged_kv_append and the decode entry points."""

    def __init__(self, num_blocks: int, block_size: int = 16, prefix_cache: bool = False):
        self._lib = _load()
        h = ctypes.c_void_p()
        _check(self._lib.pkv_bm_create(num_blocks, block_size, int(bool(prefix_cache)), ctypes.byref(h)),
               "pkv_bm_create")
        self._h = h
        self.num_blocks, self.block_size = num_blocks, block_size

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    __del__ = close

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def add_sequence(self, seq_id: int, n_prompt_tokens: int, block_hashes=None) -> int:
        """Returns the number of prompt tokens found in the prefix cache."""
        cached = ctypes.c_int64(0)
        arr = None
        if block_hashes is not None and len(block_hashes):
            arr = (ctypes.c_uint64 * len(block_hashes))(*[int(x) & (2**64 - 1) for x in block_hashes])
        _check(self._lib.pkv_bm_add_sequence(self._h, seq_id, n_prompt_tokens, arr, ctypes.byref(cached)),
               "pkv_bm_add_sequence")
        return int(cached.value)

    def fork(self, parent: int, child: int) -> None:
        _check(self._lib.pkv_bm_fork(self._h, parent, child), "pkv_bm_fork")

    def append(self, seq_ids):
        """One new token for each sequence: returns (slot_mapping int64,
        cow_src int32, cow_dst int32), host tensors."""
        ids = _host(seq_ids, torch.int64, "seq_ids").reshape(-1)
        n = ids.numel()
        slots = torch.empty(n, dtype=torch.int64)
        src = torch.empty(max(n, 1), dtype=torch.int32)
        dst = torch.empty(max(n, 1), dtype=torch.int32)
        ncow = ctypes.c_int32(0)
        _check(self._lib.pkv_bm_append(self._h, ids.data_ptr() if n else None, n,
                                       slots.data_ptr() if n else None, src.data_ptr(), dst.data_ptr(),
                                       ctypes.byref(ncow)), "pkv_bm_append")
        k = ncow.value
        return slots, src[:k].clone(), dst[:k].clone()

    def free(self, seq_id: int) -> None:
        _check(self._lib.pkv_bm_free(self._h, seq_id), "pkv_bm_free")

    def tables(self, seq_ids, width: int):
        """(block_tables int32 [n, width] with -1 padding, context_lens int32 [n]) on the host."""
        ids = _host(seq_ids, torch.int64, "seq_ids").reshape(-1)
        n = ids.numel()
        bt = torch.empty((n, width), dtype=torch.int32)
        cl = torch.empty(n, dtype=torch.int32)
        if n:
            _check(self._lib.pkv_bm_get_tables(self._h, ids.data_ptr(), n, width, bt.data_ptr(), cl.data_ptr()),
                   "pkv_bm_get_tables")
        return bt, cl

    def stats(self) -> dict:
        st = _BMStats()
        _check(self._lib.pkv_bm_stats(self._h, ctypes.byref(st)), "pkv_bm_stats")
        return {name: int(getattr(st, name)) for name, _ in _BMStats._fields_}

    def refcount(self, block: int) -> int:
        rc = ctypes.c_int32(0)
        _check(self._lib.pkv_bm_refcount(self._h, block, ctypes.byref(rc)), "pkv_bm_refcount")
        return int(rc.value)


def int8_cache(num_blocks: int, n_kv_heads: int, head_dim: int, device="cuda"):
    """An empty INT8 cache: uint8 ``[num_blocks, n_kv, 32 * head_dim + 128]``,
    one record per (block, kv head) (layout in include/pagedkv.h)."""
    return torch.zeros((num_blocks, n_kv_heads, 32 * head_dim + 128), dtype=torch.uint8, device=device)


def paged_kv_append_int8(k, v, slot_mapping, kv_cache, block_size: int = 16, stream=None) -> None:
    """Quantise ``k[i]``, ``v[i]`` into slot ``slot_mapping[i]`` of the INT8 cache (in place)."""
    lib = _load()
    num_blocks, n_kv, rb = kv_cache.shape
    d = k.shape[-1]
    if kv_cache.dtype != torch.uint8 or rb != 32 * d + 128 or k.shape[1] != n_kv:
        raise ValueError("INT8 cache shape disagrees with k")
    if v.dtype != k.dtype or slot_mapping.dtype != torch.int64:
        raise ValueError("dtype mismatch (slot_mapping must be int64)")
    if tuple(v.shape) != tuple(k.shape) or slot_mapping.shape[0] != k.shape[0]:
        raise ValueError("k, v must be [num_tokens, n_kv_heads, head_dim] and slot_mapping [num_tokens]")
    _same_device(kv_cache.device, k, v, slot_mapping)
    with torch.cuda.device(kv_cache.device):
        _check(lib.paged_kv_append_int8(_dev(k, "k"), _dev(v, "v"), _DTYPE[k.dtype],
                                        _dev(slot_mapping, "slot_mapping"), k.shape[0], _dev(kv_cache, "kv_cache"),
                                        num_blocks, block_size, n_kv, d, _stream(stream, kv_cache.device)),
               "paged_kv_append_int8")


def paged_attention_decode_int8(q, kv_cache, block_tables, context_lens, scale: float, out=None, workspace=None,
                                block_size: int = 16, stream=None):
    """paged_attention_decode over the INT8 cache; returns ``out`` (dtype of q)."""
    lib = _load()
    B, n_q, d = q.shape
    num_blocks, n_kv, rb = kv_cache.shape
    if rb != 32 * d + 128 or kv_cache.dtype != torch.uint8:
        raise ValueError("INT8 cache shape disagrees with q")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if out is None:
        out = torch.empty_like(q)
    if out.dtype != q.dtype or tuple(out.shape) != tuple(q.shape) or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor of q's dtype and shape")
    _same_device(q.device, kv_cache, out, block_tables, context_lens, workspace)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    with torch.cuda.device(q.device):
        _check(lib.paged_attention_decode_int8(
            _dev(q, "q"), _dev(kv_cache, "kv_cache"), _dev(block_tables, "block_tables"), block_tables.shape[1],
            _dev(context_lens, "context_lens"), B, num_blocks, float(scale), n_q, n_kv, d, block_size,
            _dev(out, "out"), _DTYPE[q.dtype], ws_ptr, ws_bytes, _stream(stream, q.device)),
            "paged_attention_decode_int8")
    return out


def paged_attention_mq_workspace_size(batch: int, q_len: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                                      dtype: torch.dtype) -> int:
    out = ctypes.c_size_t(0)
    _check(_load().paged_attention_mq_workspace_size(batch, q_len, n_q_heads, n_kv_heads, head_dim, _DTYPE[dtype],
                                                     ctypes.byref(out)), "paged_attention_mq_workspace_size")
    return int(out.value)


def paged_attention_decode_mq(q, k_cache, v_cache, block_tables, context_lens, scale: float, out=None,
                              workspace=None, block_size: int = 16, stream=None):
    """Several queries per sequence: ``q`` ``[batch, q_len, n_q, d]``; query i
    of a sequence sees its context up to position ``ctx - q_len + i``.
    Returns ``out`` (shape and dtype of q)."""
    lib = _load()
    B, q_len, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_cache.shape
    if d2 != d or bs != block_size or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if out is None:
        out = torch.empty_like(q)
    _check_decode_io(q, k_cache, v_cache, out, block_tables, context_lens, workspace)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    with torch.cuda.device(q.device):
        _check(lib.paged_attention_decode_mq(
            _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(block_tables, "block_tables"),
            block_tables.shape[1], _dev(context_lens, "context_lens"), B, q_len, num_blocks, float(scale), n_q,
            n_kv, d, bs, _dev(out, "out"), _DTYPE[q.dtype], ws_ptr, ws_bytes, _stream(stream, q.device)),
            "paged_attention_decode_mq")
    return out
