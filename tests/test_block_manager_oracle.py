"""The block-manager reference model against its pins, and planted mistakes
in a copy of its source that the pins must catch."""

import importlib.util
from pathlib import Path

import pytest

import oracle.block_manager as model
from tests.bm_pins import PINS

SRC = Path(model.__file__).read_text()


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(model)


# (name, text in the model's source, replacement)
MUTANTS = [
    ("no_copy_on_write", "elif self.refcount[table[-1]] > 1:\n                old", "elif False:\n                old"),
    ("evict_most_recent", "b = self.idle.pop(0)", "b = self.idle.pop()"),
    ("fork_without_refcount", "        for b in self.tables[child]:\n            self.refcount[b] += 1\n", ""),
    ("free_in_table_order", "for b in reversed(table):", "for b in table:"),
    ("highest_free_block", "b = free[0]", "b = free[-1]"),
    ("cache_hits_anywhere", "                if keys[i] not in self.block_of_key:\n                    break\n",
     "                if keys[i] not in self.block_of_key:\n                    continue\n"),
    ("new_block_one_early", "if offset == 0:", "if offset == self.block_size - 1:"),
    ("fnv_prime", "FNV_PRIME = 1099511628211", "FNV_PRIME = 1099511628213"),
    ("unchained_keys", "prev = fnv1a64(data)", "fnv1a64(data); prev = seed & MASK64"),
]


def _load_mutant(tmp_path, name, old, new):
    assert SRC.count(old) == 1, f"mutation target for {name} not found exactly once"
    path = tmp_path / f"bm_{name}.py"
    path.write_text(SRC.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"bm_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    mod = _load_mutant(tmp_path, name, old, new)
    failed = []
    for pin in PINS:
        try:
            pin(mod)
        except Exception as e:  # noqa: BLE001 - any failure of a pin counts
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"mutant {name} passed every pin"
