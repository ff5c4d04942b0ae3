"""The oracle's FP8 K/V cache path against its pins, and planted mistakes caught by them (CPU only)."""
import os

import pytest

import oracle
from tests import oracle_fp8_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "attn_oracle.c")


@pytest.mark.parametrize("pin", oracle_fp8_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


# (name, original text, replacement): each site occurs once in the oracle source.
MUTANTS = [
    ("e4m3_bias", "mag = ldexp(1.0 + (double)m / 8.0, e - 7);", "mag = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("e4m3_subnormal_scale", "mag = ldexp((double)m / 8.0, -6);", "mag = ldexp((double)m / 8.0, -7);"),
    ("e4m3_sign_dropped", "return sign ? -mag : mag;", "return mag;"),
    ("e4m3_no_nan", "if (e == 15 && m == 7)\n        return NAN;", ""),
    ("k_scale_dropped", "const double kd = e4m3_to_double(kc[(size_t)j * D + d]) * (double)ks[d];",
     "const double kd = e4m3_to_double(kc[(size_t)j * D + d]);"),
    ("v_scale_dropped", "const double vd = e4m3_to_double(vc[(size_t)j * D + d]) * (double)vs[d];",
     "const double vd = e4m3_to_double(vc[(size_t)j * D + d]);"),
    ("k_scale_one_channel", "* (double)ks[d];", "* (double)ks[0];"),
    ("k_scale_wrong_head", "k_scale + (size_t)g * D", "k_scale + (size_t)(h % Hkv) * D"),
    ("v_scale_wrong_head", "v_scale + (size_t)g * D", "v_scale + (size_t)(h % Hkv) * D"),
    ("values_from_keys", "e4m3_to_double(vc[(size_t)j * D + d])", "e4m3_to_double(kc[(size_t)j * D + d])"),
    ("mask_without_offset", "causal ? i + (Skv - Sq) + 1 : Skv;", "causal ? i + 1 : Skv;"),
    ("scores_unscaled", "sc[j] = acc * scale;", "sc[j] = acc;"),
    ("lse_without_max", "*lse_out = mx + log(den);", "*lse_out = log(den);"),
]


def _pins_that_fail(lib):
    failed = []
    for pin in oracle_fp8_pins.ALL_PINS:
        try:
            pin(lib)
        except Exception:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation site for {name} must occur once"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new), encoding="utf-8")
    lib = oracle.load(oracle.compile_oracle(str(path), str(tmp_path / f"lib{name}.so")))
    assert _pins_that_fail(lib), f"no pin caught the planted mistake {name}"
