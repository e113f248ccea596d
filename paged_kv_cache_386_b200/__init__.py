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
    "paged_kv_append", "paged_attention_decode", "paged_attention_decode_noalloc",
    "paged_attention_decode_cascade", "paged_attention_cascade_workspace_size",
    "paged_attention_workspace_size",
    "pkv_get_device_error", "pkv_status_string", "pkv_version", "PagedKVError", "library_path",
    "DEVERR_BLOCK_ID", "DEVERR_CONTEXT", "DEVERR_SLOT", "DEVERR_TIMEOUT",
]

_LIB_PATH = Path(__file__).resolve().parent / "libpagedkv.so"

PKV_F32, PKV_F16, PKV_BF16 = 0, 1, 2
_DTYPE = {torch.float32: PKV_F32, torch.float16: PKV_F16, torch.bfloat16: PKV_BF16}

PKV_OK = 0
DEVERR_BLOCK_ID, DEVERR_CONTEXT, DEVERR_SLOT, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8


class PagedKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {pkv_status_string(status)} (status {status})")


class _Options(ctypes.Structure):
    _fields_ = [("num_units", ctypes.c_int32), ("force_simt", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 6)]


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
    dec = [p, p, p, p, i32, p, i32, i32, f32, i32, i32, i32, i32, p, ctypes.c_int, p, sz, p]
    lib.paged_attention_decode.argtypes = dec
    lib.paged_attention_decode.restype = ctypes.c_int
    lib.paged_attention_decode_ex.argtypes = dec + [ctypes.POINTER(_Options)]
    lib.paged_attention_decode_ex.restype = ctypes.c_int
    lib.paged_attention_cascade_workspace_size.argtypes = [i32, i32, i32, i32, ctypes.c_int, ctypes.POINTER(sz)]
    lib.paged_attention_cascade_workspace_size.restype = ctypes.c_int
    lib.paged_attention_decode_cascade.argtypes = [p, p, p, i32, p, i32, p, p, p, i32, p, i32, i32, f32, i32, i32,
                                                   i32, i32, p, ctypes.c_int, p, sz, p]
    lib.paged_attention_decode_cascade.restype = ctypes.c_int
    lib.paged_attention_decode_noalloc.argtypes = dec[:15] + [p]
    lib.paged_attention_decode_noalloc.restype = ctypes.c_int
    lib.pkv_get_device_error.argtypes = [p, ctypes.POINTER(ctypes.c_uint32)]
    lib.pkv_get_device_error.restype = ctypes.c_int
    lib.pkv_status_string.argtypes = [ctypes.c_int]
    lib.pkv_status_string.restype = ctypes.c_char_p
    lib.pkv_version.argtypes = []
    lib.pkv_version.restype = ctypes.c_int32
    _lib = lib
    return lib


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


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
    if k.dtype != k_cache.dtype or v.dtype != k_cache.dtype or slot_mapping.dtype != torch.int64:
        raise ValueError("dtype mismatch (slot_mapping must be int64)")
    _check(lib.paged_kv_append(_dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping"),
                               k.shape[0], _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                               num_blocks, bs, n_kv, d, _DTYPE[k_cache.dtype], _stream(stream)),
           "paged_kv_append")


def paged_attention_workspace_size(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                                   dtype: torch.dtype) -> int:
    out = ctypes.c_size_t(0)
    _check(_load().paged_attention_workspace_size(batch, n_q_heads, n_kv_heads, head_dim,
                                                  _DTYPE[dtype], ctypes.byref(out)),
           "paged_attention_workspace_size")
    return int(out.value)


def paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, out=None,
                           workspace=None, num_units: int = 0, force_simt: bool = False,
                           block_size: int = 16, stream=None):
    """Single-query attention through the block table; returns ``out``."""
    lib = _load()
    B, n_q, d = q.shape
    num_blocks, n_kv, bs, d2 = k_cache.shape
    if d2 != d or bs != block_size or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if out is None:
        out = torch.empty_like(q)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    opts = _Options(num_units=int(num_units), force_simt=int(bool(force_simt)))
    _check(lib.paged_attention_decode_ex(
        _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"),
        B, num_blocks, float(scale), n_q, n_kv, d, bs, _dev(out, "out"), _DTYPE[q.dtype],
        ws_ptr, ws_bytes, _stream(stream), ctypes.byref(opts)), "paged_attention_decode")
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
                                   block_size: int = 16, stream=None):
    """Decode for sequences that share prefix blocks: group i's prefix
    (``prefix_lens[i]`` tokens in ``prefix_block_tables[i]``) is attended once
    per kv head for all its members (``seq_group[b] == i``), then each
    sequence's private suffix (``block_tables[b]``, ``context_lens[b]``
    tokens) continues from that state."""
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
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    n_groups = prefix_lens.shape[0]
    _check(lib.paged_attention_decode_cascade(
        _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), n_groups,
        _dev(prefix_block_tables, "prefix_block_tables") if n_groups else None,
        prefix_block_tables.shape[1] if n_groups else 0,
        _dev(prefix_lens, "prefix_lens") if n_groups else None, _dev(seq_group, "seq_group") if n_groups else None,
        _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"),
        B, num_blocks, float(scale), n_q, n_kv, d, bs, _dev(out, "out"), _DTYPE[q.dtype],
        ws_ptr, ws_bytes, _stream(stream)), "paged_attention_decode_cascade")
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
    _check(lib.paged_attention_decode_noalloc(
        _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"),
        B, num_blocks, float(scale), n_q, n_kv, d, bs, _dev(out, "out"), _DTYPE[q.dtype],
        _stream(stream)), "paged_attention_decode_noalloc")
    return out


def pkv_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error bits."""
    flags = ctypes.c_uint32(0)
    st = _load().pkv_get_device_error(_stream(stream), ctypes.byref(flags))
    if st not in (PKV_OK, 3):
        raise PagedKVError(st, "pkv_get_device_error")
    return int(flags.value)
