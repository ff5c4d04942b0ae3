"""The oracle's backward pass against its pins, and planted mistakes in it caught by them (CPU)."""
import os

import pytest

import oracle
from tests import oracle_bwd_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "attn_oracle.c")


@pytest.fixture(scope="module")
def lib():
    oracle.build()
    return oracle.load()


@pytest.mark.parametrize("pin", oracle_bwd_pins.BWD_PINS, ids=lambda p: p.__name__)
def test_backward_oracle_pin(lib, pin):
    pin(lib)


# (name, original text, replacement): one plausible slip each, in the backward only
MUTANTS = [
    ("d_term_dropped", "const double ds = p[j] * (dp[j] - Di);", "const double ds = p[j] * dp[j];"),
    ("d_term_sign", "const double ds = p[j] * (dp[j] - Di);", "const double ds = p[j] * (Di - dp[j]);"),
    ("dq_scale_dropped", "dq_row[d] += scale_d * ds *", "dq_row[d] += ds *"),
    ("dk_from_keys", "dk_head[(size_t)j * D + d] += scale_d * ds * bf16_to_double(q_row[d]);",
     "dk_head[(size_t)j * D + d] += scale_d * ds * bf16_to_double(k_head[(size_t)j * D + d]);"),
    ("dv_from_values", "dv_head[(size_t)j * D + d] += p[j] * bf16_to_double(do_row[d]);",
     "dv_head[(size_t)j * D + d] += p[j] * bf16_to_double(v_head[(size_t)j * D + d]);"),
    ("p_unnormalised", "p[j] = exp(s[j] - lse);", "p[j] = exp(s[j] - m);"),
    ("dp_from_keys", "dot += bf16_to_double(do_row[d]) * bf16_to_double(v_head[(size_t)j * D + d]);",
     "dot += bf16_to_double(do_row[d]) * bf16_to_double(k_head[(size_t)j * D + d]);"),
    ("mask_ignored", "const int last = causal ? i + offset : Skv - 1;", "const int last = Skv - 1;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_backward_mutant_is_caught(name, old, new, tmp_path):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation site for {name} not found"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new), encoding="utf-8")
    mlib = oracle.load(oracle.compile_oracle(str(path), str(tmp_path / f"lib{name}.so")))
    failed = []
    for pin in oracle_bwd_pins.BWD_PINS:
        try:
            pin(mlib)
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
