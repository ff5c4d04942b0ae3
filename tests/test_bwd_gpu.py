"""GPU parity of the backward pass (attn_bwd) against the fp64 oracle's gradients.

The forward runs on the GPU first (its o and lse feed the backward, as in training); the oracle
computes dq, dk, dv from q, k, v and dout alone. Tolerance: the forward's O tolerance applied to
each gradient relative to its largest magnitude — max |err| <= 1e-2 * max|ref| and
mean |err| <= 1e-3 * max|ref|. The error sources are the forward's kind: bf16 rounding of the
recomputed weights P and of dS before their tensor-core products (2^-9 relative each, fp32
accumulation), bf16 rounding of o (which enters through D_i = dO_i . O_i) and of the outputs.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_attn_b200 import attn, build, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    if torch.cuda.get_device_capability(0) != (10, 0):
        pytest.skip("needs an sm_100 device")
    build.build()
    attn.load_library()
    yield
    torch.cuda.synchronize()
    assert attn.device_status() == 0, "a kernel-side wait ran out during the backward tests"


# Shapes with fewer key tiles than SMs and an even group run each key tile as a cluster of two CTAs
# (half of the query heads each, partial dK and dV summed through distributed shared memory); the
# others one CTA per key tile.
SHAPES = [
    # B, Hq, Hkv, Sq, Skv, causal
    (1, 2, 1, 128, 128, True),    # one tile, GQA 2
    (1, 4, 2, 300, 300, True),    # ragged tails
    (2, 2, 2, 256, 384, True),    # cache offset 128
    (1, 2, 1, 200, 130, False),   # non-causal, more queries than keys
    (1, 8, 2, 512, 512, True),    # several tiles each way, GQA 4
    (1, 1, 1, 64, 1000, True),    # a short chunk over a long cache: many key tiles no row sees early
    (19, 2, 1, 1000, 1000, True),  # 152 key tiles (not fewer than the SMs): no head split, one CTA per key tile
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b{}_hq{}_hkv{}_sq{}_skv{}_{}".format(*s[:5], "c" if s[5] else "nc"))
def test_backward_matches_oracle(shape):
    B, Hq, Hkv, Sq, Skv, causal = shape
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, 128, causal, seed=sum(shape[:5]))
    q, k, v = inputs.generate(w)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    qg, kg, vg, dg = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = attn.attn_fwd(qg, kg, vg, scale=w.scale, causal=causal)
    dq, dk, dv = attn.attn_bwd(qg, kg, vg, o, lse, dg, scale=w.scale, causal=causal)
    torch.cuda.synchronize()
    ref = oracle.attention_bwd(q, k, v, dout, w.scale, causal)
    for name, got, want in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2])):
        g = got.cpu().double().numpy()
        err = np.abs(g - want)
        top = np.abs(want).max()
        assert np.isfinite(g).all(), name
        assert err.max() <= 1e-2 * top and err.mean() <= 1e-3 * top, (
            f"{name}: max|err| {err.max():.3e} mean|err| {err.mean():.3e} vs max|ref| {top:.3e}")


def test_backward_reads_and_writes_only_in_bounds():
    """q, k, v, o, dout and lse inside NaN-filled buffers, dq, dk, dv inside sentinel-filled ones:
    no NaN may leak into the gradients (nothing outside the tensors is read, ragged tails included)
    and the sentinels must survive (nothing is written out of bounds)."""
    B, Hq, Hkv, Sq, Skv = 1, 4, 2, 300, 300
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, 128, True, seed=sum((B, Hq, Hkv, Sq, Skv)))
    q, k, v = inputs.generate(w)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    pad = 4096

    def inside(t, fill):
        buf = torch.full((2 * pad + t.numel(),), fill, dtype=t.dtype, device="cuda")
        buf[pad:pad + t.numel()] = t.reshape(-1).to("cuda")
        return buf, buf[pad:pad + t.numel()].view(t.shape)

    nan = float("nan")
    _, qd = inside(q, nan)
    _, kd = inside(k, nan)
    _, vd = inside(v, nan)
    _, dd = inside(dout, nan)
    o, lse = attn.attn_fwd(qd, kd, vd, scale=w.scale, causal=True)
    _, od = inside(o, nan)
    _, lsed = inside(lse, nan)
    bufs = [inside(torch.full(t.shape, 7.0, dtype=torch.bfloat16), 7.0) for t in (q, k, v)]
    attn.attn_bwd(qd, kd, vd, od, lsed, dd, scale=w.scale, causal=True, dq=bufs[0][1], dk=bufs[1][1], dv=bufs[2][1])
    torch.cuda.synchronize()
    ref = oracle.attention_bwd(q, k, v, dout, w.scale, True)
    for (buf, view), want, name in zip(bufs, ref, ("dq", "dk", "dv")):
        n = view.numel()
        assert (buf[:pad] == 7.0).all() and (buf[pad + n:] == 7.0).all(), name
        g = view.cpu().double().numpy()
        assert np.isfinite(g).all(), name
        err = np.abs(g - want)
        top = np.abs(want).max()
        assert err.max() <= 1e-2 * top and err.mean() <= 1e-3 * top, name
