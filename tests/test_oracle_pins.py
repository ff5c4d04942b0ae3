"""The CPU oracle against the pages' worked examples, closed forms, invariants and a brute force."""
import math

import pytest

from tests import oracle_pins
from causal_attention_attn_b200 import inputs


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_head_dim_scale_matches_page():
    """1/scale for D = 128 is sqrt(128) ~ 11.3 ("Vì sao chia cho √128")."""
    g = oracle_pins.GOLDEN["sqrt_head_dim"]
    assert abs(1.0 / inputs.PREFILL_8B.scale - g["sqrt_d"]) <= g["printed_tolerance"]
    assert abs(inputs.PREFILL_8B.scale - 1.0 / math.sqrt(128)) < 1e-8


def test_rejects_causal_with_more_queries_than_keys(oracle_lib):
    q, k, v = oracle_pins.rand_qkv(1, 1, 1, 5, 4, 4, seed=1)
    import oracle

    with pytest.raises(ValueError):
        oracle.attention(q, k, v, 0.5, causal=True, lib=oracle_lib)
    oracle.attention(q, k, v, 0.5, causal=False, lib=oracle_lib)
