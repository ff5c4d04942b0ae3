"""GPU parity of the single-token decode over an FP8 (e4m3) K/V cache — attn_decode_fp8 and
attn_decode_paged_fp8 — against the fp64 oracle over the dequantised cache.

The cache is the seeded bf16 cache quantised per (kv head, channel) (``inputs.generate_fp8``); the
oracle decodes the same codes and coefficients. Tolerance: the decode's own (O max |err| <= 1e-2,
mean <= 1e-3; LSE max |err| <= 1e-3). The kernel's extra error over the bf16 path is the 3-part
e4m3 split of q * k_scale and of the weights (about 2^-12 relative each), well inside it.
"""
import numpy as np
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
    assert attn.device_status() == 0, "a kernel-side wait ran out during the fp8 decode tests"


def run(q, k8, v8, ks, vs, scale, ctas=0):
    o, lse = attn.attn_decode_fp8(q.cuda(), k8.cuda(), v8.cuda(), ks.cuda(), vs.cuda(), scale=scale,
                                  decode_ctas=ctas)
    torch.cuda.synchronize()
    return o, lse


SHAPES = [
    # B, Hq, Hkv, Skv, decode_ctas
    (2, 8, 2, 300, 0),      # 4 heads per kv head, ragged last chunk
    (3, 4, 4, 129, 0),      # one head per kv head
    (2, 32, 2, 700, 0),     # 16 heads per kv head
    (2, 6, 2, 257, 0),      # group of 3: one head per pair
    (1, 16, 2, 1, 0),       # a single cached key
    (2, 8, 2, 1000, 5),     # pairs shared by CTAs: partials merged
    (2, 8, 2, 1000, 37),
    (1, 8, 1, 64, 300),     # more CTAs than chunks
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b{}_hq{}_hkv{}_skv{}_ctas{}".format(*s))
def test_fp8_decode_matches_oracle(shape):
    B, Hq, Hkv, Skv, ctas = shape
    w = inputs.custom(B, Hq, Hkv, 1, Skv, 128, True, seed=Skv + 17 * Hq)
    q, k8, v8, ks, vs = inputs.generate_fp8(w)
    o, lse = run(q, k8, v8, ks, vs, w.scale, ctas)
    ro, rl = oracle.attention_fp8kv(q, k8, v8, ks, vs, w.scale, True)
    rep = compare(o, lse, ro, rl)
    assert rep.ok(), str(rep)


def test_fp8_decode_workload_full():
    """The bench's decode shape (B=16, Hq=32, Hkv=8, Skv=4096) in e4m3, every row against the oracle."""
    w = inputs.DECODE_GQA
    q, k8, v8, ks, vs = inputs.generate_fp8(w)
    o, lse = run(q, k8, v8, ks, vs, w.scale)
    ro, rl = oracle.attention_fp8kv(q, k8, v8, ks, vs, w.scale, True)
    rep = compare(o, lse, ro, rl)
    assert rep.ok(), str(rep)


def test_fp8_channel_coefficients_are_used_per_kv_head():
    """Distinct, non-uniform coefficients per (kv head, channel): a mix-up of heads or channels fails.
    V's coefficients stay below 0.0052 so that |v~| <= 2.4 and O keeps the unit scale the absolute
    tolerance is stated for (at |O| ~ 600 the bf16 rounding of O alone exceeds 1e-2)."""
    w = inputs.custom(2, 8, 2, 1, 384, 128, True, seed=99)
    q, k8, v8, _, _ = inputs.generate_fp8(w)
    g = torch.Generator().manual_seed(3)
    ks = torch.rand((2, 128), generator=g) * 0.05 + 0.001
    vs = torch.rand((2, 128), generator=g) * 0.005 + 0.0002
    o, lse = run(q, k8, v8, ks, vs, w.scale)
    ro, rl = oracle.attention_fp8kv(q, k8, v8, ks, vs, w.scale, True)
    rep = compare(o, lse, ro, rl)
    assert rep.ok(), str(rep)


def test_fp8_decode_with_large_and_tiny_queries():
    """q * k_scale far above and far below 1 (q scaled by 4096 and by 1/4096, the softmax scale by the
    inverse, so the scores keep their size): the per-head power of two moves the split to the top of
    the e4m3 range either way."""
    w = inputs.custom(2, 8, 2, 1, 256, 128, True, seed=5)
    q, k8, v8, ks, vs = inputs.generate_fp8(w)
    for factor in (4096.0, 1.0 / 4096.0):
        qf = (q.float() * factor).to(torch.bfloat16)  # exact: a power of two
        scale = float(torch.tensor(w.scale / factor, dtype=torch.float32))
        o, lse = run(qf, k8, v8, ks, vs, scale)
        ro, rl = oracle.attention_fp8kv(qf, k8, v8, ks, vs, scale, True)
        rep = compare(o, lse, ro, rl)
        assert rep.ok(), f"factor {factor}: {rep}"


def make_paged_fp8(w, lens, page_size, seed):
    q, k8, v8, ks, vs = inputs.generate_fp8(w)
    B, Hkv, cap, D = k8.shape
    pages_per_seq = -(-cap // page_size)
    num_pages = B * pages_per_seq + 3
    rng = np.random.RandomState(seed)
    perm = rng.permutation(num_pages)
    table = np.full((B, pages_per_seq), num_pages + 7, dtype=np.int32)
    kp = torch.full((num_pages, Hkv, page_size, D), E4M3_NAN, dtype=torch.uint8)  # unused slots: NaN codes
    vp = kp.clone()
    nxt = 0
    for b in range(B):
        for n in range(-(-lens[b] // page_size)):
            pg = int(perm[nxt])
            nxt += 1
            table[b, n] = pg
            lo, hi = n * page_size, min((n + 1) * page_size, lens[b])
            kp[pg, :, : hi - lo] = k8[b, :, lo:hi]
            vp[pg, :, : hi - lo] = v8[b, :, lo:hi]
    return q, k8, v8, ks, vs, kp, vp, torch.from_numpy(table), torch.tensor(lens, dtype=torch.int32)


PAGED = [
    # B, Hq, Hkv, capacity, page_size, lengths, decode_ctas
    (4, 32, 8, 1000, 64, [1000, 1, 129, 0], 0),
    (3, 8, 8, 700, 16, [700, 127, 128], 0),
    (2, 32, 2, 300, 128, [300, 256], 5),
    (6, 8, 2, 64, 32, [64, 64, 1, 0, 33, 63], 300),
]


@pytest.mark.parametrize("case", PAGED, ids=lambda c: "b{}_hq{}_hkv{}_cap{}_page{}_ctas{}".format(*c[:5], c[6]))
def test_paged_fp8_decode_matches_oracle(case):
    B, Hq, Hkv, cap, page_size, lens, ctas = case
    w = inputs.custom(B, Hq, Hkv, 1, cap, 128, True, seed=sum(lens) + page_size + 1)
    q, k8, v8, ks, vs, kp, vp, table, seq_lens = make_paged_fp8(w, lens, page_size, seed=B + cap)
    o, lse = attn.attn_decode_paged_fp8(q.cuda(), kp.cuda(), vp.cuda(), ks.cuda(), vs.cuda(), table.cuda(),
                                        seq_lens.cuda(), max(lens), scale=w.scale, decode_ctas=ctas)
    torch.cuda.synchronize()
    o, lse = o.cpu(), lse.cpu()
    for b in range(B):
        if lens[b] == 0:
            assert torch.all(o[b].float() == 0) and torch.all(torch.isneginf(lse[b])), b
            continue
        n = lens[b]
        ro, rl = oracle.attention_fp8kv(q[b:b + 1], k8[b:b + 1, :, :n].contiguous(), v8[b:b + 1, :, :n].contiguous(),
                                        ks, vs, w.scale, True)
        rep = compare(o[b:b + 1], lse[b:b + 1], ro, rl)
        if n == 1:
            # One key: O is that key's dequantised value row itself, which bf16 cannot hold exactly
            # (a code times an fp32 coefficient); its correct rounding alone averages ~1e-3 for
            # N(0, 1)-sized values, the mean bound itself. Required instead: O is the correctly
            # rounded value (at most half a bf16 ulp away) and the LSE bound.
            assert rep.o_max_ulps <= 0.5 + 1e-6 and rep.lse_max_abs <= 1e-3, f"batch {b} (length 1): {rep}"
            continue
        assert rep.ok(), f"batch {b} (length {n}): {rep}"


def test_fp8_decode_reads_and_writes_only_in_bounds():
    """The e4m3 cache sits inside buffers of NaN codes and the coefficient tables inside NaN floats;
    O and LSE inside sentinel-filled buffers: no NaN may leak in (nothing past Skv or past the
    tables is read) and the sentinels must survive (nothing is written out of bounds)."""
    B, Hq, Hkv, Skv = 1, 4, 2, 333
    w = inputs.custom(B, Hq, Hkv, 1, Skv, 128, True, seed=333)
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
    lbuf, ld = inside(torch.full((B, Hq, 1), 7.0), 7.0)
    attn.attn_decode_fp8(q.cuda(), kd, vd, ksd, vsd, scale=w.scale, out=od, lse=ld)
    torch.cuda.synchronize()
    assert torch.isfinite(od.float()).all() and torch.isfinite(ld).all()
    assert (obuf[:pad] == 7.0).all() and (obuf[pad + q.numel():] == 7.0).all()
    assert (lbuf[:pad] == 7.0).all() and (lbuf[pad + B * Hq:] == 7.0).all()
    rep = compare(od, ld, *oracle.attention_fp8kv(q, k8, v8, ks, vs, w.scale, True))
    assert rep.ok(), str(rep)
