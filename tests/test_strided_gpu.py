"""GPU parity of attention over strided layouts (``attn_fwd_strided`` through the binding's views)
against the fp64 oracle: token-major [B, S, H, D] tensors, q, k and v as head slices of one fused
[B, S, Hq + 2*Hkv, D] projection output, mixed layouts, and an output written in token-major order.

The oracle takes the same values in the heads-major layout (a plain permutation of the same
elements), so any mistake in a stride, a coordinate or the output addressing shows up as a
mismatch. Tolerance (tests/compare.py): O max|err| <= 1e-2, mean|err| <= 1e-3; LSE max|err| <= 1e-3.
"""
import pytest
import torch

import oracle
from causal_attention_attn_b200 import attn, build, inputs
from tests.compare import compare

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
    assert attn.device_status() == 0, "a kernel-side wait ran out during the strided-layout tests"


def token_major(x):
    """The [B, S, H, D] copy of a heads-major tensor, returned as its [B, H, S, D] view."""
    return x.transpose(1, 2).contiguous().cuda().transpose(1, 2)


SHAPES = [
    # B, Hq, Hkv, Sq, Skv, D, causal
    (2, 8, 2, 300, 300, 128, True),
    (1, 4, 4, 130, 700, 128, True),     # cache offset 570
    (2, 6, 2, 200, 200, 64, True),      # odd group: consecutive query tiles per CTA
    (1, 4, 1, 257, 300, 32, False),
    (3, 32, 8, 1, 1000, 128, True),     # decode, tensor core
    (2, 8, 8, 1, 333, 64, True),        # decode with D 64: runs the prefill kernel
    (2, 6, 3, 1, 129, 32, True),        # decode with D 32: runs the prefill kernel
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b{}_hq{}_hkv{}_sq{}_skv{}_d{}_{}".format(
    *s[:6], "c" if s[6] else "nc"))
def test_token_major_layout_matches_oracle(shape):
    B, Hq, Hkv, Sq, Skv, D, causal = shape
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, D, causal, seed=sum(shape[:6]) + 5)
    q, k, v = inputs.generate(w)
    out = torch.full((B, Sq, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    o, lse = attn.attn_fwd(token_major(q), token_major(k), token_major(v), scale=w.scale, causal=causal, out=out)
    torch.cuda.synchronize()
    assert o.data_ptr() == out.data_ptr()
    rep = compare(o, lse, *oracle.attention(q, k, v, w.scale, causal))
    assert rep.ok(), str(rep)


@pytest.mark.parametrize("Sq,D", [(384, 128), (1, 128), (200, 64)])
def test_fused_qkv_projection_slices(Sq, D):
    """q, k, v as head slices of one [B, S, Hq + 2*Hkv, D] buffer (the output of a fused QKV
    projection), read without copies; the output goes to a heads-major tensor."""
    B, Hq, Hkv = 2, 8, 2
    w = inputs.custom(B, Hq, Hkv, Sq, Sq, D, True, seed=Sq + D)
    q, k, v = inputs.generate(w)
    qkv = torch.cat([x.transpose(1, 2) for x in (q, k, v)], dim=2).contiguous().cuda()  # [B, S, Hq+2Hkv, D]
    qv = qkv[:, :, :Hq].transpose(1, 2)
    kv = qkv[:, :, Hq:Hq + Hkv].transpose(1, 2)
    vv = qkv[:, :, Hq + Hkv:].transpose(1, 2)
    assert not qv.is_contiguous()
    o, lse = attn.attn_fwd(qv, kv, vv, scale=w.scale, causal=True)
    torch.cuda.synchronize()
    rep = compare(o, lse, *oracle.attention(q, k, v, w.scale, True))
    assert rep.ok(), str(rep)


def test_mixed_layouts_and_strided_output_agree_with_contiguous_call_bitwise():
    """The layout changes only the addresses: a token-major q with heads-major k, v and a
    token-major output gives the same bits as the contiguous call."""
    w = inputs.custom(1, 8, 2, 333, 333, 128, True, seed=21)
    q, k, v = inputs.generate(w)
    o_ref, l_ref = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=w.scale, causal=True)
    out = torch.empty((1, 333, 8, 128), dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    o, lse = attn.attn_fwd(token_major(q), k.cuda(), v.cuda(), scale=w.scale, causal=True, out=out)
    torch.cuda.synchronize()
    assert torch.equal(o.contiguous(), o_ref) and torch.equal(lse, l_ref)


def test_strided_reads_and_writes_stay_in_bounds():
    """A fused QKV buffer inside NaN padding and a token-major output inside sentinel padding: no
    NaN may leak in and every sentinel must survive, for a prefill and a decode."""
    B, Hq, Hkv, S, D, pad = 1, 4, 2, 200, 128, 8192
    w = inputs.custom(B, Hq, Hkv, S, S, D, True, seed=33)
    q, k, v = inputs.generate(w)
    H = Hq + 2 * Hkv
    n = B * S * H * D
    buf = torch.full((2 * pad + n,), float("nan"), dtype=torch.bfloat16, device="cuda")
    buf[pad:pad + n] = torch.cat([x.transpose(1, 2) for x in (q, k, v)], dim=2).reshape(-1).cuda()
    qkv = buf[pad:pad + n].view(B, S, H, D)
    for sq in (S, 1):
        qv = qkv[:, S - sq:, :Hq].transpose(1, 2)
        kv, vv = qkv[:, :, Hq:Hq + Hkv].transpose(1, 2), qkv[:, :, Hq + Hkv:].transpose(1, 2)
        m = B * sq * Hq * D
        obuf = torch.full((2 * pad + m,), 7.0, dtype=torch.bfloat16, device="cuda")
        out = obuf[pad:pad + m].view(B, sq, Hq, D).transpose(1, 2)
        o, lse = attn.attn_fwd(qv, kv, vv, scale=w.scale, causal=True, out=out)
        torch.cuda.synchronize()
        assert (obuf[:pad] == 7.0).all() and (obuf[pad + m:] == 7.0).all()
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        rep = compare(o, lse, *oracle.attention(q[:, :, S - sq:].contiguous(), k, v, w.scale, True))
        assert rep.ok(), f"sq={sq}: {rep}"
