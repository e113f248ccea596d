"""The oracle's multi-query decode against its pins, and planted mistakes in
that part of the oracle's C source that the pins must catch."""

from pathlib import Path

import pytest

import oracle
from tests.oracle_mq_pins import PINS

SRC = Path(oracle.__file__).resolve().parent / "pkv_oracle.c"


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(oracle.load())


MUTANTS = [
    ("causal_limit_off_by_one", "int32_t ctx_i = context_lens[b] - q_len + i + 1;",
     "int32_t ctx_i = context_lens[b] - q_len + i;"),
    ("no_causal_limit", "int32_t ctx_i = context_lens[b] - q_len + i + 1;", "int32_t ctx_i = context_lens[b];"),
    ("query_row_transposed", "const char* q_row = (const char*)q + ((size_t)b * q_len + i) * n_q_heads * head_dim * es;",
     "const char* q_row = (const char*)q + ((size_t)i * batch + b) * n_q_heads * head_dim * es;"),
    ("short_context_accepted", "if (context_lens[b] < q_len) {", "if (context_lens[b] < 0) {"),
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
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
