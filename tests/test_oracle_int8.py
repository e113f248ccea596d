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
    ("k_not_swizzled", "return (size_t)j * d + (size_t)((c ^ (j % (chunks < 8 ? chunks : 8))) * 16 + e % 16);",
     "return (size_t)j * d + (size_t)(c * 16 + e % 16);"),
    ("v_scale_from_k", "memcpy(&vsf, rec + (size_t)32 * d + 64 + 4 * off, 4);", "memcpy(&vsf, rec + (size_t)32 * d + 4 * off, 4);"),
    ("amax_signed", "float a = fabsf(x);", "float a = x;"),
    ("v_row_stride", "rec[(size_t)16 * head_dim + (size_t)e * 16 + vpos(off)] = (uint8_t)codes[e];",
     "rec[(size_t)16 * head_dim + (size_t)e * 8 + vpos(off)] = (uint8_t)codes[e];"),
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
