"""Pins for the oracle's FP8 (e4m3) K/V cache path, each against something other than the
oracle's fp8 code itself: torch's e4m3 conversion, values worked out from the format's definition,
the bf16 oracle (pinned on its own in ``oracle_pins.py``), exact power-of-two scaling identities,
and the closed form for a zero query.

Sources: "MLA 矩阵乘法吸收的数值稳定性治理", §五 (FP8 cache, higher-precision accumulation) and
§二.1 (a coefficient per feature channel). Every pin takes the oracle library as its argument so
that the mutant tests can run it against a planted mistake.
"""
import numpy as np
import torch

import oracle


def _codes(shape, seed):
    """Random finite e4m3 codes (NaN codes 0x7f and 0xff replaced by 0x7e)."""
    g = torch.Generator().manual_seed(seed)
    c = torch.randint(0, 256, shape, generator=g, dtype=torch.int64).to(torch.uint8)
    c[(c == 0x7F) | (c == 0xFF)] = 0x7E
    return c


def _dec_torch(codes):
    return codes.view(torch.float8_e4m3fn).to(torch.float64)


def _q(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def pin_decoder_matches_torch(lib):
    codes = torch.arange(256, dtype=torch.int64).to(torch.uint8)
    got = oracle.decode_e4m3(codes, lib=lib)
    want = _dec_torch(codes).numpy()
    nan = np.isnan(want)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def pin_decoder_named_values(lib):
    # From the definition: bias 7, three mantissa bits, e = 0 subnormal with scale 2^-6.
    table = {0x00: 0.0, 0x38: 1.0, 0xB8: -1.0, 0x3C: 1.5, 0x30: 0.5, 0x7E: 448.0, 0xFE: -448.0,
             0x08: 2.0 ** -6, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x40: 2.0, 0x77: 240.0}
    codes = np.array(list(table), dtype=np.uint8)
    got = oracle.decode_e4m3(codes, lib=lib)
    assert np.array_equal(got, np.array(list(table.values())))
    assert np.signbit(oracle.decode_e4m3(np.array([0x80], dtype=np.uint8), lib=lib)[0])


def _bf16_of_codes(codes):
    # every e4m3 value is exactly a bf16 value
    return codes.view(torch.float8_e4m3fn).to(torch.bfloat16)


def pin_unit_scales_equal_bf16_oracle(lib):
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 2, 5, 9, 16
    q = _q((B, Hq, Sq, D), 1)
    k8, v8 = _codes((B, Hkv, Skv, D), 2), _codes((B, Hkv, Skv, D), 3)
    ones = np.ones((Hkv, D), dtype=np.float32)
    for causal in (True, False):
        o8, l8 = oracle.attention_fp8kv(q, k8, v8, ones, ones, 0.125, causal, lib=lib)
        o, l = oracle.attention(q, _bf16_of_codes(k8), _bf16_of_codes(v8), 0.125, causal)
        assert np.array_equal(o8, o) and np.array_equal(l8, l)


def pin_v_channel_scales_scale_outputs(lib):
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 2, 3, 7, 8
    q = _q((B, Hq, Sq, D), 4)
    k8, v8 = _codes((B, Hkv, Skv, D), 5), _codes((B, Hkv, Skv, D), 6)
    ones = np.ones((Hkv, D), dtype=np.float32)
    vs = np.array([[2.0 ** ((d % 5) - 2 + 3 * g) for d in range(D)] for g in range(Hkv)], dtype=np.float32)
    o1, l1 = oracle.attention_fp8kv(q, k8, v8, ones, ones, 0.3, True, lib=lib)
    o2, l2 = oracle.attention_fp8kv(q, k8, v8, ones, vs, 0.3, True, lib=lib)
    per_head = vs[np.arange(Hq) // (Hq // Hkv)]  # [Hq, D]
    assert np.array_equal(o2, o1 * per_head[None, :, None, :]) and np.array_equal(l2, l1)


def pin_k_channel_scales_fold_into_q(lib):
    # sum_d q_d (k_d s_d) == sum_d (q_d s_d) k_d exactly for power-of-two s_d
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 2, 4, 6, 8
    q = _q((B, Hq, Sq, D), 7)
    k8, v8 = _codes((B, Hkv, Skv, D), 8), _codes((B, Hkv, Skv, D), 9)
    ones = np.ones((Hkv, D), dtype=np.float32)
    ks = np.array([[2.0 ** (((d + 2 * g) % 4) - 2) for d in range(D)] for g in range(Hkv)], dtype=np.float32)
    o8, l8 = oracle.attention_fp8kv(q, k8, v8, ks, ones, 0.07, True, lib=lib)
    q_scaled = (q.double() * torch.from_numpy(ks[np.arange(Hq) // (Hq // Hkv)]).double()[None, :, None, :]).to(torch.bfloat16)
    assert torch.equal(q_scaled.double(), q.double() * torch.from_numpy(ks[np.arange(Hq) // (Hq // Hkv)]).double()[None, :, None, :])
    o, l = oracle.attention(q_scaled, _bf16_of_codes(k8), _bf16_of_codes(v8), 0.07, True)
    assert np.array_equal(o8, o) and np.array_equal(l8, l)


def pin_zero_query_closed_form(lib):
    # q = 0: every visible key has weight 1/n, so o = mean of the dequantised visible values and
    # lse = ln n, with n = i + (Skv - Sq) + 1 under the cache-aligned causal mask.
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 3, 8, 4
    q = torch.zeros((B, Hq, Sq, D), dtype=torch.bfloat16)
    k8, v8 = _codes((B, Hkv, Skv, D), 10), _codes((B, Hkv, Skv, D), 11)
    ks = np.full((Hkv, D), 0.5, dtype=np.float32)
    vs = np.array([[0.25, 1.0, 3.0, 0.125]], dtype=np.float32)
    o, l = oracle.attention_fp8kv(q, k8, v8, ks, vs, 1.0, True, lib=lib)
    vdq = _dec_torch(v8).numpy() * vs[0]  # [B, Hkv, Skv, D]
    for i in range(Sq):
        n = i + (Skv - Sq) + 1
        want = vdq[0, 0, :n].mean(axis=0)
        for h in range(Hq):
            assert np.allclose(o[0, h, i], want, rtol=1e-14, atol=1e-15)
            assert abs(l[0, h, i] - np.log(n)) < 1e-14


ALL_PINS = [pin_decoder_matches_torch, pin_decoder_named_values, pin_unit_scales_equal_bf16_oracle,
            pin_v_channel_scales_scale_outputs, pin_k_channel_scales_fold_into_q, pin_zero_query_closed_form]
