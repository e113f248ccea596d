"""Planted mistakes in the oracle's C source (compiled on the CPU into a
temporary library) must each fail at least one pin.  This shows the pins are
strong enough to catch a dropped term, a wrong sign, a wrong index or a
swapped operand in the oracle."""

from pathlib import Path

import pytest

import oracle
from tests.oracle_pins import PINS

SRC = Path(oracle.__file__).resolve().parent / "pkv_oracle.c"

# (name, text in the oracle source, replacement)
MUTANTS = [
    ("dropped_scale", "s[j] = scale * acc;", "s[j] = acc;"),
    ("gqa_modulo_mapping", "int32_t kvh = h / group;", "int32_t kvh = h % n_kv;"),
    ("block_index_uses_offset", "max_blocks_per_seq + j / bs];", "max_blocks_per_seq + j % bs];"),
    ("slot_offset_uses_block", "kvh) * bs + (j % bs))", "kvh) * bs + (j / bs) % bs)"),
    ("context_off_by_one", "int32_t ctx = context_lens[b];", "int32_t ctx = context_lens[b] - (context_lens[b] > 1);"),
    ("softmax_sign_flip", "s[j] = exp(s[j] - m);", "s[j] = exp(m - s[j]);"),
    ("k_for_v_in_sum", "out_row[e] += s[j] * V[(size_t)j * d + e];", "out_row[e] += s[j] * K[(size_t)j * d + e];"),
    ("no_normalisation", "out_row[e] /= denom;", "out_row[e] /= 1.0;"),
    ("token_major_block_layout", "(((size_t)phys * n_kv + kvh) * bs + (j % bs))", "(((size_t)phys * bs + (j % bs)) * n_kv + kvh)"),
    ("query_row_of_kv_head", "((size_t)b * n_q + h) * d + e", "((size_t)b * n_q + kvh) * d + e"),
    ("append_head_stride", "size_t dst = (((size_t)blk * n_kv_heads + h) * block_size + off) * row;",
     "size_t dst = (((size_t)blk * block_size + off) * n_kv_heads + h) * row;"),
    ("f16_exponent_bias", "expo - 25", "expo - 24"),
    ("f16_subnormal_scale", "ldexp((double)frac, -24)", "ldexp((double)frac, -25)"),
    ("bf16_low_half", "uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h << 15;"),
    ("f16_sign_dropped", "return sign ? -mag : mag;", "return mag;"),
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
        except Exception:  # an assertion, an oracle error or a NaN reaching the brute force
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
