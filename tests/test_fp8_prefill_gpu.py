"""GPU parity of attn_prefill_fp8 (prefill of Sq queries over an FP8 (e4m3) K/V cache with fp32
per-(kv head, channel) coefficients) against the fp64 oracle over the dequantised cache.

The cache is the seeded bf16 cache quantised per (kv head, channel) (``inputs.generate_fp8``); the
oracle decodes the same codes and coefficients. Tolerance: the forward's (O max |err| <= 1e-2, mean
<= 1e-3; LSE max |err| <= 1e-3). The kernel's extra error over the bf16 path is the 3-part e4m3
split of q * k_scale (about 2^-12 relative); the weights' 2-part split (about 2^-8) matches the
bf16 rounding of the weights in the bf16 path.
"""
import pytest
import torch

import oracle
from causal_attention_attn_b200 import attn, build, inputs
from tests.compare import compare

pytestmark = pytest.mark.gpu

E4M3_NAN = 0x7F


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
    assert attn.device_status() == 0, "a kernel-side wait ran out during the fp8 prefill tests"


def run(q, k8, v8, ks, vs, scale, causal=True):
    o, lse = attn.attn_prefill_fp8(q.cuda(), k8.cuda(), v8.cuda(), ks.cuda(), vs.cuda(), scale=scale, causal=causal)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


SHAPES = [
    # B, Hq, Hkv, Sq, Skv, causal
    (2, 8, 2, 256, 768, True),     # chunked prefill over a cached prefix
    (1, 4, 1, 300, 300, True),     # plain causal prefill, ragged last tiles (row 0 sees one key)
    (2, 6, 2, 130, 513, True),     # odd group, ragged query and key tiles
    (1, 8, 8, 64, 1000, False),    # non-causal, one query tile, eight KV tiles
    (3, 4, 2, 1, 257, True),       # a single query row per head
    (1, 32, 8, 384, 384, True),    # 8B-layer head structure
    (2, 4, 4, 300, 100, False),    # non-causal with more queries than keys, one partial KV tile
    (1, 2, 2, 17, 17, True),       # tiny: one partial query tile and one partial KV tile
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b{}_hq{}_hkv{}_sq{}_skv{}_{}".format(
    *s[:5], "c" if s[5] else "nc"))
def test_fp8_prefill_matches_oracle(shape):
    B, Hq, Hkv, Sq, Skv, causal = shape
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, 128, causal, seed=Skv + 31 * Sq + Hq)
    q, k8, v8, ks, vs = inputs.generate_fp8(w)
    o, lse = run(q, k8, v8, ks, vs, w.scale, causal)
    ro, rl = oracle.attention_fp8kv(q, k8, v8, ks, vs, w.scale, causal)
    rep = compare(o, lse, ro, rl)
    assert rep.ok(), str(rep)


def test_fp8_prefill_chunked_workload_sampled_rows():
    """The bench's chunked-prefill shape (B8 Hq32 Hkv8, 256 new tokens over 768 cached) in e4m3,
    a deterministic sample of rows covering every (b, head) against the oracle."""
    w = inputs.CHUNKED_PREFILL
    q, k8, v8, ks, vs = inputs.generate_fp8(w)
    o, lse = run(q, k8, v8, ks, vs, w.scale, True)
    rows = inputs.sample_rows(w, every=16)
    ro, rl = oracle.attention_fp8kv(q, k8, v8, ks, vs, w.scale, True, rows=rows.numpy())
    rep = compare(o.reshape(-1, 128)[rows], lse.reshape(-1)[rows], ro, rl)
    assert rep.ok(), str(rep)


def test_fp8_prefill_channel_coefficients_and_query_range():
    """Distinct coefficients per (kv head, channel), and q scaled far above and below 1 (the softmax
    scale by the inverse): the per-row power of two keeps the split at the top of the e4m3 range."""
    w = inputs.custom(2, 8, 2, 200, 460, 128, True, seed=77)
    q, k8, v8, _, _ = inputs.generate_fp8(w)
    g = torch.Generator().manual_seed(4)
    ks = torch.rand((2, 128), generator=g) * 0.05 + 0.001
    vs = torch.rand((2, 128), generator=g) * 0.005 + 0.0002
    for factor in (1.0, 4096.0, 1.0 / 4096.0):
        qf = (q.float() * factor).to(torch.bfloat16)  # exact: a power of two
        scale = float(torch.tensor(w.scale / factor, dtype=torch.float32))
        o, lse = run(qf, k8, v8, ks, vs, scale, True)
        rep = compare(o, lse, *oracle.attention_fp8kv(qf, k8, v8, ks, vs, scale, True))
        assert rep.ok(), f"factor {factor}: {rep}"


def test_fp8_prefill_reads_and_writes_only_in_bounds():
    """The cache inside buffers of NaN codes, the coefficient tables inside NaN floats, O and LSE
    inside sentinel-filled buffers: no NaN leaks in, every sentinel survives."""
    B, Hq, Hkv, Sq, Skv = 1, 4, 2, 150, 333
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, 128, True, seed=334)
    q, k8, v8, ks, vs = inputs.generate_fp8(w)
    pad = 4096

    def inside(t, fill):
        buf = torch.full((2 * pad + t.numel(),), fill, dtype=t.dtype, device="cuda")
        buf[pad:pad + t.numel()] = t.reshape(-1).cuda()
        return buf, buf[pad:pad + t.numel()].view(t.shape)

    _, kd = inside(k8, E4M3_NAN)
    _, vd = inside(v8, E4M3_NAN)
    _, ksd = inside(ks, float("nan"))
    _, vsd = inside(vs, float("nan"))
    obuf, od = inside(torch.full(q.shape, 7.0, dtype=torch.bfloat16), 7.0)
    lbuf, ld = inside(torch.full((B, Hq, Sq), 7.0), 7.0)
    attn.attn_prefill_fp8(q.cuda(), kd, vd, ksd, vsd, scale=w.scale, out=od, lse=ld)
    torch.cuda.synchronize()
    assert torch.isfinite(od.float()).all() and torch.isfinite(ld).all()
    assert (obuf[:pad] == 7.0).all() and (obuf[pad + q.numel():] == 7.0).all()
    assert (lbuf[:pad] == 7.0).all() and (lbuf[pad + B * Hq * Sq:] == 7.0).all()
    rep = compare(od.cpu(), ld.cpu(), *oracle.attention_fp8kv(q, k8, v8, ks, vs, w.scale, True))
    assert rep.ok(), str(rep)
