"""The C-ABI library loads without a GPU, exports every entry point that
include/pagedkv.h declares, and rejects bad arguments on the host before
touching CUDA (no compute call is made here)."""

import ctypes
import re
from pathlib import Path

import pytest

import paged_kv_cache_386_b200 as pkv
from paged_kv_cache_386_b200 import build as pkv_build

HEADER = Path(__file__).resolve().parents[1] / "include" / "pagedkv.h"

INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 5


@pytest.fixture(scope="module")
def lib():
    pkv_build.build()
    return pkv._load()


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)


def test_header_declares_expected_entry_points():
    names = set(declared_functions())
    assert {"paged_kv_append", "paged_attention_decode", "paged_attention_decode_ex",
            "paged_attention_workspace_size", "pkv_get_device_error", "pkv_status_string",
            "pkv_version", "paged_kv_copy_blocks", "paged_attention_workspace_size_ex", "pkv_bm_create", "pkv_bm_destroy", "pkv_bm_hash_blocks",
            "pkv_bm_add_sequence", "pkv_bm_fork", "pkv_bm_append", "pkv_bm_free", "pkv_bm_get_tables",
            "pkv_bm_stats", "pkv_bm_refcount", "paged_kv_append_and_decode"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(8):
        assert pkv.pkv_status_string(s)
    assert pkv.pkv_status_string(99) == "unknown status"
    assert pkv.pkv_version() >= 10000


def _decode(lib, **over):
    args = dict(q=None, k=None, v=None, bt=None, maxb=4, cl=None, batch=2, nblocks=8, scale=0.125,
                nq=8, nkv=2, d=128, bs=16, out=None, dtype=2, ws=None, wsb=0, stream=None)
    args.update(over)
    a = args
    return lib.paged_attention_decode(a["q"], a["k"], a["v"], a["bt"], a["maxb"], a["cl"], a["batch"],
                                      a["nblocks"], a["scale"], a["nq"], a["nkv"], a["d"], a["bs"],
                                      a["out"], a["dtype"], a["ws"], a["wsb"], a["stream"])


def test_decode_host_validation(lib):
    assert _decode(lib) == INVALID                      # null pointers
    assert _decode(lib, nq=6, nkv=4) == INVALID          # n_q % n_kv != 0
    assert _decode(lib, batch=-1) == INVALID
    assert _decode(lib, nblocks=0) == INVALID
    assert _decode(lib, scale=float("nan")) == INVALID
    assert _decode(lib, d=96) == UNSUPPORTED
    assert _decode(lib, bs=32) == UNSUPPORTED
    assert _decode(lib, dtype=7) == UNSUPPORTED
    assert _decode(lib, batch=4097) == UNSUPPORTED
    assert _decode(lib, batch=0) == 0                    # nothing to do, nothing enqueued
    # misaligned q (pointers are never dereferenced on the host)
    assert _decode(lib, q=8, k=256, v=512, bt=1024, cl=2048, out=4096) == INVALID
    # tile count beyond 32 bits
    assert _decode(lib, q=256, k=256, v=256, bt=256, cl=256, out=256, batch=4096, maxb=1 << 20) == UNSUPPORTED


def test_decode_ex_rejects_bad_options(lib):
    opts = pkv._Options(num_units=-1)
    st = lib.paged_attention_decode_ex(256, 256, 256, 256, 4, 256, 2, 8, 0.1, 8, 2, 128, 16, 256, 2,
                                       None, 0, None, ctypes.byref(opts))
    assert st == INVALID
    for bad in (dict(reserved=(ctypes.c_int32 * 2)(0, 1)), dict(balance_chunks=5), dict(balance_chunks=-1),
                dict(static_permille=100), dict(static_permille=1000), dict(wait_limit_us=-5),
                dict(test_withhold_unit=-2)):
        opts = pkv._Options(**bad)
        st = lib.paged_attention_decode_ex(256, 256, 256, 256, 4, 256, 2, 8, 0.1, 8, 2, 128, 16, 256, 2,
                                           None, 0, None, ctypes.byref(opts))
        assert st == INVALID, bad


def test_fused_append_and_decode_host_validation(lib):
    f = lib.paged_kv_append_and_decode
    ptr = 256

    def call(q=ptr, k=ptr, v=ptr, sl=ptr, ntok=2, kc=ptr, vc=ptr, bt=ptr, maxb=4, cl=ptr, batch=2, nb=8,
             scale=0.125, nq=8, nkv=2, d=128, bs=16, out=ptr, dtype=2):
        return f(q, k, v, sl, ntok, kc, vc, bt, maxb, cl, batch, nb, scale, nq, nkv, d, bs, out, dtype, None, 0, None)

    assert call(ntok=-1) == INVALID                      # the append's checks
    assert call(k=None) == INVALID
    assert call(sl=260) == INVALID                       # slot_mapping misaligned
    assert call(bs=32) == UNSUPPORTED
    assert call(nq=6, nkv=4) == INVALID                  # the decode's checks
    assert call(q=8) == INVALID
    assert call(d=96) == UNSUPPORTED
    assert call(scale=float("nan")) == INVALID


def test_append_host_validation(lib):
    f = lib.paged_kv_append
    assert f(None, None, None, -1, None, None, 8, 16, 2, 128, 2, None) == INVALID
    assert f(None, None, None, 4, None, None, 8, 32, 2, 128, 2, None) == UNSUPPORTED
    assert f(None, None, None, 4, None, None, 8, 16, 2, 128, 9, None) == UNSUPPORTED
    assert f(None, None, None, 0, None, None, 8, 16, 2, 128, 2, None) == 0
    assert f(None, None, None, 4, None, None, 8, 16, 2, 128, 2, None) == INVALID
    assert f(16, 32, 4, 4, 64, 128, 8, 16, 2, 128, 2, None) == INVALID   # slot_mapping misaligned


def test_copy_blocks_host_validation(lib):
    f = lib.paged_kv_copy_blocks
    assert f(None, None, None, None, -1, 8, 16, 2, 128, 2, None) == INVALID
    assert f(None, None, None, None, 4, 8, 32, 2, 128, 2, None) == UNSUPPORTED
    assert f(None, None, None, None, 4, 8, 16, 2, 128, 7, None) == UNSUPPORTED
    assert f(None, None, None, None, 0, 8, 16, 2, 128, 2, None) == 0
    assert f(None, None, None, None, 4, 8, 16, 2, 128, 2, None) == INVALID
    assert f(16, 32, 2, 64, 4, 8, 16, 2, 128, 2, None) == INVALID       # src_blocks misaligned


def test_workspace_size_validation(lib):
    out = ctypes.c_size_t()
    assert lib.paged_attention_workspace_size(4, 6, 4, 128, 2, ctypes.byref(out)) == INVALID
    assert lib.paged_attention_workspace_size(4, 8, 2, 96, 2, ctypes.byref(out)) == UNSUPPORTED
    assert lib.paged_attention_workspace_size(4, 8, 2, 128, 2, None) == INVALID


def test_device_error_needs_flags(lib):
    assert lib.pkv_get_device_error(None, None) == INVALID


def test_binding_rejects_cpu_tensors():
    import torch
    t = torch.zeros(1, 8, 128, dtype=torch.bfloat16)
    cache = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pkv.paged_attention_decode(t, cache, cache, torch.zeros(1, 1, dtype=torch.int32),
                                   torch.ones(1, dtype=torch.int32), 0.1, out=t.clone())


def test_cascade_options_are_checked_on_the_host(lib):
    ptr = ctypes.c_void_p(16)  # never dereferenced: the options are rejected first
    for fields in ({"prefix_splits": 5}, {"prefix_splits": -1}, {"prefix_kernel": 3}):
        opts = pkv._CascadeOptions(**fields)
        st = lib.paged_attention_decode_cascade_ex(ptr, ptr, ptr, 1, ptr, 4, ptr, ptr, ptr, 4, ptr, 2, 8, 0.125,
                                                   8, 2, 128, 16, ptr, 2, None, 0, None, ctypes.byref(opts))
        assert st == INVALID, fields
    opts = pkv._CascadeOptions()
    opts.reserved[3] = 1
    st = lib.paged_attention_decode_cascade_ex(ptr, ptr, ptr, 1, ptr, 4, ptr, ptr, ptr, 4, ptr, 2, 8, 0.125,
                                               8, 2, 128, 16, ptr, 2, None, 0, None, ctypes.byref(opts))
    assert st == INVALID


def test_header_compiles_as_plain_c(tmp_path):
    # The boundary is a C ABI: the header must stand alone in strict C99.
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    src = tmp_path / "uses_header.c"
    src.write_text('#include "pagedkv.h"\n'
                   "int main(void) {\n"
                   "  pkv_decode_options d = {0};\n"
                   "  pkv_cascade_options c = {0};\n"
                   "  pkv_bm_stats_t s;\n"
                   "  (void)d; (void)c; (void)s;\n"
                   "  return PKV_OK;\n"
                   "}\n")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                        "-I", str(HEADER.parent), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_binding_checks_dtypes_and_shapes_before_any_cuda_call(lib):
    # The C layer sees raw pointers and q's dtype only; the binding refuses
    # caches or outputs of another dtype or shape (CPU tensors suffice: the
    # checks run before any pointer is taken).
    import torch
    q = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    kc = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16)
    bt = torch.zeros(2, 2, dtype=torch.int32)
    cl = torch.ones(2, dtype=torch.int32)
    with pytest.raises(ValueError, match="dtype"):
        pkv.paged_attention_decode(q, kc.half(), kc.half(), bt, cl, 0.1)
    with pytest.raises(ValueError, match="out"):
        pkv.paged_attention_decode(q, kc, kc, bt, cl, 0.1, out=torch.zeros(2, 8, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out"):
        pkv.paged_attention_decode(q, kc, kc, bt, cl, 0.1, out=torch.zeros(2, 8, 128, dtype=torch.float16))
    with pytest.raises(ValueError, match="out"):
        pkv.paged_attention_decode_noalloc(q, kc, kc, bt, cl, 0.1, out=torch.zeros(3, 8, 128, dtype=torch.bfloat16))
    k = torch.zeros(2, 2, 128, dtype=torch.bfloat16)
    sl = torch.zeros(2, dtype=torch.int64)
    with pytest.raises(ValueError):
        pkv.paged_kv_append_and_decode(q, k.half(), k.half(), sl, kc, kc, bt, cl, 0.1)
    with pytest.raises(ValueError):
        pkv.paged_kv_append(k[:, :1], k[:, :1], sl, kc, kc)   # wrong kv-head count
