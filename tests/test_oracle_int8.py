"""The oracle's INT8 cache against its pins, and planted mistakes in the INT8
part of the oracle's C source (compiled on the CPU into temporary libraries)
that the pins must catch."""

from pathlib import Path

import pytest

import oracle
from tests.oracle_int8_pins import PINS

SRC = Path(oracle.__file__).resolve().parent / "pkv_oracle.c"


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(oracle.load())


MUTANTS = [
    ("scale_128", "float scale = amax / 127.0f;", "float scale = amax / 128.0f;"),
    ("truncating_codes", "rintf(x / scale)", "truncf(x / scale)"),
    ("round_half_away", "rintf(x / scale)", "roundf(x / scale)"),
    ("vpos_swapped_halves", "return 4 * ((j % 8) / 2) + 2 * (j / 8) + (j % 2);",
     "return 2 * ((j % 8) / 2) + 8 * (j / 8) + (j % 2);"),
    ("v_not_transposed_on_read", "V[(size_t)j * d + e] = vs * (double)v8[(bh * d + e) * bs + vpos(off)];",
     "V[(size_t)j * d + e] = vs * (double)v8[(bh * bs + off) * d + e];"),
    ("k_scale_for_v", "double ks = (double)k_scale[bh * bs + off], vs = (double)v_scale[bh * bs + off];",
     "double ks = (double)k_scale[bh * bs + off], vs = (double)k_scale[bh * bs + off];"),
    ("k_row_offset", "memcpy(k8 + (bh * block_size + off) * head_dim", "memcpy(k8 + (bh * block_size + (off ^ 1)) * head_dim"),
    ("amax_signed", "float a = fabsf(x);", "float a = x;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    text = SRC.read_text()
    assert text.count(old) == 1, f"mutation target for {name} not found exactly once"
    src = tmp_path / f"{name}.c"
    src.write_text(text.replace(old, new))
    lib = oracle.load(oracle.build(src, tmp_path / f"lib{name}.so"))
    failed = []
    for pin in PINS:
        try:
            pin(lib)
        except Exception:  # an assertion or an oracle error
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
