"""Pins for the oracle's backward pass (gradients of a loss through the attention), independent of
the oracle's own code. Each pin takes the loaded oracle library, so that planted mistakes in the
oracle can be shown to be caught (tests/test_oracle_bwd_pins.py).

Kinds of pin:
  * numerical derivative: central differences of an independent numpy forward (a materialised
    score matrix with an explicit cache-aligned mask, softmax, weighted sum of V) on tiny shapes,
    for every element of q, k and v;
  * the exact derivative: torch autograd in fp64 through a materialised forward (score matrix,
    explicit cache-aligned mask, softmax, weighted sum of V), written independently of the oracle;
  * invariants that follow from the softmax: every row of dS sums to zero, so the key gradients sum
    to zero and a shift of every key by the same vector changes no gradient; every row of P sums to
    one, so the value gradients sum to the sum of dO over the rows that read them.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _numpy_forward(q, k, v, scale, causal):
    """O for fp64 q [B,Hq,Sq,D], k/v [B,Hkv,Skv,D]: the plain matrix form with an explicit mask."""
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    out = np.zeros_like(q)
    i = np.arange(Sq)[:, None]
    j = np.arange(Skv)[None, :]
    visible = (j <= i + (Skv - Sq)) if causal else np.ones((Sq, Skv), dtype=bool)
    for b in range(B):
        for h in range(Hq):
            s = scale * q[b, h] @ k[b, h // g].T
            s = np.where(visible, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[b, h] = p @ v[b, h // g]
    return out


def _fd_check(lib, B, Hq, Hkv, Sq, Skv, D, causal, seed):
    q = _rand_bf16((B, Hq, Sq, D), seed)
    k = _rand_bf16((B, Hkv, Skv, D), seed + 1)
    v = _rand_bf16((B, Hkv, Skv, D), seed + 2)
    do = _rand_bf16((B, Hq, Sq, D), seed + 3)
    scale = float(np.float32(D ** -0.5))
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale, causal, lib=lib)
    qd, kd, vd, dod = (t.float().double().numpy() for t in (q, k, v, do))

    def loss(qq, kk, vv):
        return float((_numpy_forward(qq, kk, vv, scale, causal) * dod).sum())

    eps = 1e-5
    for name, x, grad in (("dq", qd, dq), ("dk", kd, dk), ("dv", vd, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"dq": (xp, kd, vd), "dk": (qd, xp, vd), "dv": (qd, kd, xp)}[name]
            args_m = {"dq": (xm, kd, vd), "dk": (qd, xm, vd), "dv": (qd, kd, xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        err = np.abs(num - grad).max()
        assert err < 1e-7, f"{name}: finite differences disagree by {err:.3e}"


def pin_bwd_finite_differences_causal_gqa(lib):
    _fd_check(lib, 1, 2, 1, 3, 5, 4, True, seed=11)  # cache offset 2, two query heads per kv head


def pin_bwd_finite_differences_noncausal(lib):
    _fd_check(lib, 2, 2, 2, 4, 3, 4, False, seed=21)  # more queries than keys, two batches


def pin_bwd_finite_differences_square_causal(lib):
    _fd_check(lib, 1, 1, 1, 4, 4, 3, True, seed=31)


def _medium(seed, causal=True):
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 2, 7, 11, 8
    q = _rand_bf16((B, Hq, Sq, D), seed)
    k = _rand_bf16((B, Hkv, Skv, D), seed + 1)
    v = _rand_bf16((B, Hkv, Skv, D), seed + 2)
    do = _rand_bf16((B, Hq, Sq, D), seed + 3)
    return q, k, v, do, float(np.float32(D ** -0.5)), causal


def pin_bwd_key_gradients_sum_to_zero(lib):
    for causal in (True, False):
        q, k, v, do, scale, _ = _medium(41, causal)
        _, dk, _ = oracle.attention_bwd(q, k, v, do, scale, causal, lib=lib)
        assert np.abs(dk.sum(axis=2)).max() < 1e-12


def pin_bwd_value_gradients_sum_to_dout(lib):
    # sum_j dV_j = sum over the group's rows i of dO_i (each row of P sums to one)
    q, k, v, do, scale, causal = _medium(51)
    _, _, dv = oracle.attention_bwd(q, k, v, do, scale, causal, lib=lib)
    B, Hq, Sq, D = q.shape
    Hkv = k.shape[1]
    dod = do.float().double().numpy().reshape(B, Hkv, Hq // Hkv, Sq, D)
    assert np.abs(dv.sum(axis=2) - dod.sum(axis=(2, 3))).max() < 1e-12


def pin_bwd_key_shift_changes_nothing(lib):
    # Keys on a grid of 1/8 shifted by the same vector (exact in bf16): every gradient is unchanged.
    rng = np.random.RandomState(61)
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 5, 6, 4
    q = _bf16(rng.randint(-16, 17, size=(B, Hq, Sq, D)) / 8.0)
    k = rng.randint(-64, 65, size=(B, Hkv, Skv, D)) / 8.0
    u = rng.randint(-16, 17, size=(D,)) / 8.0
    v = _bf16(rng.randint(-16, 17, size=(B, Hkv, Skv, D)) / 8.0)
    do = _bf16(rng.randint(-16, 17, size=(B, Hq, Sq, D)) / 8.0)
    scale = 0.5
    g0 = oracle.attention_bwd(q, _bf16(k), v, do, scale, True, lib=lib)
    g1 = oracle.attention_bwd(q, _bf16(k + u), v, do, scale, True, lib=lib)
    for a, b in zip(g0, g1):
        assert np.abs(a - b).max() < 1e-12


def _autograd_check(lib, B, Hq, Hkv, Sq, Skv, D, causal, seed):
    q = _rand_bf16((B, Hq, Sq, D), seed)
    k = _rand_bf16((B, Hkv, Skv, D), seed + 1)
    v = _rand_bf16((B, Hkv, Skv, D), seed + 2)
    do = _rand_bf16((B, Hq, Sq, D), seed + 3)
    scale = float(np.float32(D ** -0.5))
    got = oracle.attention_bwd(q, k, v, do, scale, causal, lib=lib)
    qt, kt, vt = (t.double().requires_grad_(True) for t in (q, k, v))
    g = Hq // Hkv
    kr, vr = kt.repeat_interleave(g, dim=1), vt.repeat_interleave(g, dim=1)  # query head h reads kv head h // g
    s = scale * qt @ kr.transpose(-1, -2)
    i = torch.arange(Sq)[:, None]
    j = torch.arange(Skv)[None, :]
    visible = (j <= i + (Skv - Sq)) if causal else torch.ones((Sq, Skv), dtype=torch.bool)
    p = torch.softmax(s.masked_fill(~visible, float("-inf")), dim=-1)
    ((p @ vr) * do.double()).sum().backward()
    for name, mine, ref in zip(("dq", "dk", "dv"), got, (qt.grad, kt.grad, vt.grad)):
        err = np.abs(mine - ref.numpy()).max()
        assert err <= 1e-12 * max(1.0, np.abs(ref.numpy()).max()), (name, err)


def pin_bwd_autograd_causal_gqa_cached(lib):
    # GQA group 3, a cache offset of 5 (Sq = 7 over Skv = 12), causal
    _autograd_check(lib, 2, 6, 2, 7, 12, 16, True, seed=71)


def pin_bwd_autograd_noncausal_more_queries(lib):
    _autograd_check(lib, 1, 4, 1, 9, 5, 8, False, seed=81)


BWD_PINS = [
    pin_bwd_autograd_causal_gqa_cached,
    pin_bwd_autograd_noncausal_more_queries,
    pin_bwd_finite_differences_causal_gqa,
    pin_bwd_finite_differences_noncausal,
    pin_bwd_finite_differences_square_causal,
    pin_bwd_key_gradients_sum_to_zero,
    pin_bwd_value_gradients_sum_to_dout,
    pin_bwd_key_shift_changes_nothing,
]
