"""Pins for the CPU oracle: checks against what the pages and the mathematics fix, independent of
the oracle's own code. Each pin takes the loaded oracle library so that the mutation test can run
the same pins against deliberately broken builds and show that every planted mistake is caught.

Kinds of pin used here:
  * values the pages print for worked examples (``tests/golden/pages_worked_examples.json``);
  * closed forms (zero queries -> prefix mean of V and LSE = ln(count));
  * invariants the pages state (shift invariance, masked keys get weight exactly 0, earlier rows
    never change when tokens are appended, decode needs no mask);
  * a library-routine brute force (scipy softmax/logsumexp over a materialised score matrix with an
    explicit mask built the way the cache-aligned mask is described).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import scipy.special
import torch

import oracle

GOLDEN = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                     "pages_worked_examples.json"), encoding="utf-8"))


def bf16(x) -> torch.Tensor:
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def bf16_exact(values) -> bool:
    t = torch.tensor(values, dtype=torch.float64)
    return bool(torch.equal(t.to(torch.bfloat16).to(torch.float64), t))


def score_probe(lib, key_rows, q_vec, scale=1.0):
    """One query over len(key_rows) keys with V = identity rows, so O equals the softmax weights.

    q_vec and every key row have the same length D_s; D = max(D_s, n) and the remaining
    coordinates are zero. Returns (weights[n], lse) in float64.
    """
    n = len(key_rows)
    ds = len(q_vec)
    D = max(ds, n)
    q = np.zeros((1, 1, 1, D), np.float32)
    q[0, 0, 0, :ds] = q_vec
    k = np.zeros((1, 1, n, D), np.float32)
    for j, row in enumerate(key_rows):
        k[0, 0, j, :ds] = row
    v = np.zeros((1, 1, n, D), np.float32)
    for j in range(n):
        v[0, 0, j, j] = 1.0
    o, lse = oracle.attention(bf16(q), bf16(k), bf16(v), scale, causal=False, lib=lib)
    return o[0, 0, 0, :n], float(lse[0, 0, 0])


def rand_qkv(B, Hq, Hkv, Sq, Skv, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, Sq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, Skv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, Skv, D), generator=g).to(torch.bfloat16)
    return q, k, v


# ---------------------------------------------------------------------------------------------
# Values printed on the pages
# ---------------------------------------------------------------------------------------------

def pin_dot_product(lib):
    """(2,-1,0.5).(3,4,2) = 3: with one key and scale 1 the LSE is the score itself."""
    g = GOLDEN["dot_product"]
    v = [1.0, -2.0, 0.25]
    q = bf16(np.array(g["q"]).reshape(1, 1, 1, 3))
    k = bf16(np.array(g["k"]).reshape(1, 1, 1, 3))
    o, lse = oracle.attention(q, k, bf16(np.array(v).reshape(1, 1, 1, 3)), 1.0, causal=True, lib=lib)
    assert float(lse[0, 0, 0]) == float(g["value"]), lse
    assert np.array_equal(o[0, 0, 0], np.array(v)), o


def pin_softmax_printed(lib):
    """softmax(2, 1, 0.1) -> e^x = 7.39, 2.72, 1.11 (sum 11.2) -> 66%, 24%, 10%."""
    g = GOLDEN["softmax_three_scores"]
    w, lse = score_probe(lib, [[s] for s in g["scores"]], [1.0])
    assert np.allclose(w, g["weights"], atol=g["printed_tolerance_weights"], rtol=0), w
    assert abs(math.exp(lse) - g["exp_sum"]) <= g["printed_tolerance_sum"], lse
    exps = w * math.exp(lse)
    assert np.allclose(exps, g["exp_values"], atol=g["printed_tolerance_exp"], rtol=0), exps
    assert abs(w.sum() - 1.0) < 1e-15


def pin_shift_printed(lib):
    """Subtracting the row max (2;1;0.1 -> 0;-1;-1.9) leaves the weights as printed."""
    g = GOLDEN["softmax_shifted_scores"]
    w, _ = score_probe(lib, [[s] for s in g["scores"]], [1.0])
    assert np.allclose(w, g["weights"], atol=g["printed_tolerance_weights"], rtol=0), w


def pin_shift_exact(lib):
    """softmax(x - c) = softmax(x) exactly (bf16-exact scores), and LSE shifts by c."""
    x = [2.0, 1.0, 0.125]
    xs = [a - 2.0 for a in x]
    assert bf16_exact(x) and bf16_exact(xs)
    w1, l1 = score_probe(lib, [[s] for s in x], [1.0])
    w2, l2 = score_probe(lib, [[s] for s in xs], [1.0])
    assert np.max(np.abs(w1 - w2)) < 1e-15, (w1, w2)
    assert abs((l1 - l2) - 2.0) < 1e-14, (l1, l2)


def pin_large_scores(lib):
    """Scores near 1026 overflow exp() unless the row max is subtracted first."""
    x = [2.0, 1.0, 0.125]
    w_ref, l_ref = score_probe(lib, [[s] for s in x], [1.0])
    w, lse = score_probe(lib, [[1024.0, s] for s in x], [1.0, 1.0])
    assert np.all(np.isfinite(w)) and math.isfinite(lse), (w, lse)
    assert np.max(np.abs(w - w_ref)) < 1e-12, (w, w_ref)
    assert abs(lse - (1024.0 + l_ref)) < 1e-10, (lse, l_ref)


def pin_online_blocks(lib):
    """Blocks [2,1] then [3,0]: the running sum with the final max 3 is ~1.55, and merging the two
    blocks' LSEs gives the whole row's LSE."""
    g = GOLDEN["online_softmax_blocks"]
    row = [s for blk in g["blocks"] for s in blk]
    _, lse = score_probe(lib, [[s] for s in row], [1.0])
    m = max(row)
    assert abs(math.exp(lse - m) - g["running_sum"]) <= g["printed_tolerance"], lse
    parts = [score_probe(lib, [[s] for s in blk], [1.0])[1] for blk in g["blocks"]]
    assert abs(np.logaddexp(*parts) - lse) < 1e-12, (parts, lse)


# ---------------------------------------------------------------------------------------------
# Causal mask and KV cache invariants
# ---------------------------------------------------------------------------------------------

def pin_causal_row0(lib):
    """Row 0 sees only key 0: O[0] = V[0] exactly; with V = 1 every row's weights sum to 1."""
    q, k, v = rand_qkv(1, 2, 2, 16, 16, 8, seed=11)
    o, lse = oracle.attention(q, k, v, 0.35, causal=True, lib=lib)
    assert np.array_equal(o[:, :, 0, :], v[:, :, 0, :].double().numpy())
    dot00 = (q[:, :, 0, :].double() * k[:, :, 0, :].double()).sum(-1).numpy()
    assert np.allclose(lse[:, :, 0], float(np.float32(0.35)) * dot00, atol=1e-12)
    ones = torch.ones_like(v)
    o1, _ = oracle.attention(q, k, ones, 0.35, causal=True, lib=lib)
    assert np.max(np.abs(o1 - 1.0)) < 1e-13


def pin_future_keys_ignored(lib):
    """A masked key gets weight exactly 0: changing keys/values in a row's future changes nothing."""
    q, k, v = rand_qkv(1, 1, 1, 8, 8, 4, seed=12)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 5:, :] = 30.0
    v2[:, :, 5:, :] = -100.0
    o1, l1 = oracle.attention(q, k, v, 0.5, causal=True, lib=lib)
    o2, l2 = oracle.attention(q, k2, v2, 0.5, causal=True, lib=lib)
    assert np.array_equal(o1[:, :, :5], o2[:, :, :5]) and np.array_equal(l1[:, :, :5], l2[:, :, :5])
    assert not np.array_equal(o1[:, :, 5:], o2[:, :, 5:])


def pin_zero_query_closed_form(lib):
    """q = 0 makes every visible score 0: O_i = mean of V over the visible prefix and LSE = ln(count).
    Cache-aligned mask: query i of Sq sees keys 0 .. i + (Skv - Sq)."""
    B, H, Sq, Skv, D = 1, 2, 5, 9, 4
    _, k, v = rand_qkv(B, H, H, Sq, Skv, D, seed=13)
    q = torch.zeros((B, H, Sq, D), dtype=torch.bfloat16)
    o, lse = oracle.attention(q, k, v, 0.5, causal=True, lib=lib)
    vd = v.double().numpy()
    for i in range(Sq):
        n = i + (Skv - Sq) + 1
        assert np.allclose(o[:, :, i], vd[:, :, :n].mean(axis=2), atol=1e-14), i
        assert np.allclose(lse[:, :, i], math.log(n), atol=1e-14), i
    o, lse = oracle.attention(q, k, v, 0.5, causal=False, lib=lib)
    assert np.allclose(o, vd.mean(axis=2, keepdims=True), atol=1e-14)
    assert np.allclose(lse, math.log(Skv), atol=1e-14)


def pin_prefix_unchanged_on_append(lib):
    """Earlier rows never change when tokens are appended (why the KV cache is exact)."""
    q, k, v = rand_qkv(1, 2, 1, 20, 20, 8, seed=14)
    o_full, l_full = oracle.attention(q, k, v, 0.3, causal=True, lib=lib)
    o_pre, l_pre = oracle.attention(q[:, :, :12], k[:, :, :12], v[:, :, :12], 0.3, causal=True, lib=lib)
    assert np.array_equal(o_full[:, :, :12], o_pre) and np.array_equal(l_full[:, :, :12], l_pre)


def pin_chunk_equals_tail_of_full(lib):
    """Sq new queries over a cache of Skv keys equal the last Sq rows of a full causal prefill."""
    q, k, v = rand_qkv(2, 2, 2, 11, 11, 8, seed=15)
    o_full, l_full = oracle.attention(q, k, v, 0.3, causal=True, lib=lib)
    o_c, l_c = oracle.attention(q[:, :, 7:], k, v, 0.3, causal=True, lib=lib)
    assert np.array_equal(o_full[:, :, 7:], o_c) and np.array_equal(l_full[:, :, 7:], l_c)


def pin_decode_is_last_row(lib):
    """One new query over the cache needs no mask: causal and non-causal agree, and both equal the
    last row of the full prefill."""
    q, k, v = rand_qkv(1, 4, 2, 9, 9, 8, seed=16)
    o_full, l_full = oracle.attention(q, k, v, 0.3, causal=True, lib=lib)
    o_c, l_c = oracle.attention(q[:, :, 8:], k, v, 0.3, causal=True, lib=lib)
    o_n, l_n = oracle.attention(q[:, :, 8:], k, v, 0.3, causal=False, lib=lib)
    assert np.array_equal(o_c, o_n) and np.array_equal(l_c, l_n)
    assert np.array_equal(o_full[:, :, 8:], o_c) and np.array_equal(l_full[:, :, 8:], l_c)


def pin_gqa_is_repeated_mha(lib):
    """Grouped heads: query head h reads kv head h // (Hq/Hkv), i.e. MHA with each K/V head repeated."""
    q, k, v = rand_qkv(2, 6, 2, 7, 10, 8, seed=17)
    o1, l1 = oracle.attention(q, k, v, 0.3, causal=True, lib=lib)
    kr = k.repeat_interleave(3, dim=1)
    vr = v.repeat_interleave(3, dim=1)
    o2, l2 = oracle.attention(q, kr, vr, 0.3, causal=True, lib=lib)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_rows_subset(lib):
    """Asking for a subset of rows returns exactly those rows of the full result."""
    q, k, v = rand_qkv(2, 4, 2, 9, 13, 8, seed=18)
    o_full, l_full = oracle.attention(q, k, v, 0.3, causal=True, lib=lib)
    rows = np.array([0, 5, 17, 35, 40, 71], dtype=np.int64)
    o_r, l_r = oracle.attention(q, k, v, 0.3, causal=True, rows=rows, lib=lib)
    assert np.array_equal(o_full.reshape(-1, 8)[rows], o_r) and np.array_equal(l_full.reshape(-1)[rows], l_r)


# ---------------------------------------------------------------------------------------------
# Brute force through library routines on a materialised score matrix
# ---------------------------------------------------------------------------------------------

def brute_force(q, k, v, scale, causal):
    """fp64 numpy: S = scale * Q K^T per head (K/V heads repeated for grouping); for causal, a
    square -inf upper triangle (diagonal excluded) is added to the LAST Sq key columns; then
    scipy softmax and logsumexp along the keys, and O = P V."""
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    B, Hq, Sq, D = qd.shape
    g = Hq // kd.shape[1]
    kd = np.repeat(kd, g, axis=1)
    vd = np.repeat(vd, g, axis=1)
    s = np.float64(np.float32(scale)) * np.einsum("bhid,bhjd->bhij", qd, kd)
    if causal:
        tri = np.triu(np.full((Sq, Sq), -np.inf), k=1)
        s[..., -Sq:] = s[..., -Sq:] + tri
    p = scipy.special.softmax(s, axis=-1)
    return np.einsum("bhij,bhjd->bhid", p, vd), scipy.special.logsumexp(s, axis=-1)


BRUTE_SHAPES = [
    # B, Hq, Hkv, Sq, Skv, D, causal
    (1, 1, 1, 1, 1, 1, True),
    (1, 2, 2, 7, 7, 5, True),
    (2, 4, 2, 5, 12, 8, True),
    (1, 6, 3, 12, 12, 16, False),
    (2, 2, 1, 3, 17, 4, False),
    (1, 8, 2, 16, 40, 32, True),
]


def pin_brute_force(lib):
    for n, (B, Hq, Hkv, Sq, Skv, D, causal) in enumerate(BRUTE_SHAPES):
        q, k, v = rand_qkv(B, Hq, Hkv, Sq, Skv, D, seed=100 + n)
        scale = 1.0 / math.sqrt(D) if D > 1 else 0.7
        o, lse = oracle.attention(q, k, v, scale, causal, lib=lib)
        o_bf, lse_bf = brute_force(q, k, v, scale, causal)
        assert np.max(np.abs(o - o_bf)) < 1e-12, (n, np.max(np.abs(o - o_bf)))
        assert np.max(np.abs(lse - lse_bf)) < 1e-12, (n, np.max(np.abs(lse - lse_bf)))


ALL_PINS = [
    pin_dot_product, pin_softmax_printed, pin_shift_printed, pin_shift_exact, pin_large_scores,
    pin_online_blocks, pin_causal_row0, pin_future_keys_ignored, pin_zero_query_closed_form,
    pin_prefix_unchanged_on_append, pin_chunk_equals_tail_of_full, pin_decode_is_last_row,
    pin_gqa_is_repeated_mha, pin_rows_subset, pin_brute_force,
]
