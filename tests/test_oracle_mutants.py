"""Planted mistakes in the oracle must be caught by the pins.

Each mutant is a copy of ``oracle/attn_oracle.c`` with one plausible slip (a dropped term, a wrong
sign or index, a transposed operand), compiled on the CPU into a temporary library. The test runs
every pin from ``tests/oracle_pins.py`` against it and requires at least one to fail, so the pins
that vouch for the oracle are shown to have teeth. Nothing here touches a GPU.
"""
import os

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "attn_oracle.c")

# (name, original text, replacement, expected number of occurrences replaced)
MUTANTS = [
    ("mask_top_left_alignment", "last_visible = causal ? i + offset : Skv - 1", "last_visible = causal ? i : Skv - 1", 1),
    ("mask_off_by_one", "last_visible = causal ? i + offset : Skv - 1",
     "last_visible = causal ? i + offset - 1 + (i == 0) : Skv - 1", 1),
    ("mask_offset_sign", "const int offset = Skv - Sq; /* the mask", "const int offset = Sq - Skv; /* the mask", 1),
    ("scale_dropped", "scores[j] = scale * dot;", "scores[j] = dot;", 1),
    ("max_not_subtracted", "l += exp(scores[j] - m);", "l += exp(scores[j]);", 1),
    ("lse_without_max", "*lse_out = m + log(l);", "*lse_out = log(l);", 1),
    ("lse_log2", "*lse_out = m + log(l);", "*lse_out = m + log2(l);", 1),
    ("no_normalisation", "double w = exp(scores[j] - m) / l;", "double w = exp(scores[j] - m);", 1),
    ("gqa_modulo_mapping", "const int kvh = h / group;", "const int kvh = h % Hkv;", 1),
    ("values_read_from_keys", "const uint16_t *v_row = v_head + (size_t)j * D;",
     "const uint16_t *v_row = k_head + (size_t)j * D;", 1),
    ("dot_wrong_index", "bf16_to_double(k_row[d]);", "bf16_to_double(k_row[0]);", 1),
    ("row_decode_swapped", "const int i = (int)(row % Sq);", "const int i = (int)(row / Sq % Sq);", 1),
    ("last_key_excluded", "for (int j = 0; j <= last_visible; ++j) {\n        double w",
     "for (int j = 0; j < last_visible; ++j) {\n        double w", 1),
]


def _pins_that_fail(lib):
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except Exception:  # an assertion, a NaN comparison, or a rejected call all count
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, count, tmp_path):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == count, f"mutation site for {name} not found in the oracle source"
    mutated = src.replace(old, new)
    path = tmp_path / f"{name}.c"
    path.write_text(mutated, encoding="utf-8")
    lib_path = oracle.compile_oracle(str(path), str(tmp_path / f"lib{name}.so"))
    failed = _pins_that_fail(oracle.load(lib_path))
    assert failed, f"no pin caught the planted mistake {name}"


def test_unmutated_oracle_passes_every_pin(oracle_lib):
    assert _pins_that_fail(oracle_lib) == []
