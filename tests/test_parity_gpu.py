"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on the same seeded
inputs, element by element, plus invariants the pages state, checked on the GPU outputs.

Tolerance (tests/compare.py): O max|err| <= 1e-2, mean|err| <= 1e-3; LSE max|err| <= 1e-3.
"""
import math

import numpy as np
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
    major, minor = torch.cuda.get_device_capability(0)
    if (major, minor) != (10, 0):
        pytest.skip("needs an sm_100 device")
    build.build()
    attn.load_library()
    yield
    torch.cuda.synchronize()
    assert attn.device_status() == 0, "a kernel-side wait ran out during the parity tests"


def run_gpu(q, k, v, scale, causal, decode_ctas=0):
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=scale, causal=causal, decode_ctas=decode_ctas)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def check(q, k, v, scale, causal, rows=None, decode_ctas=0):
    o, lse = run_gpu(q, k, v, scale, causal, decode_ctas)
    if rows is None:
        o_ref, lse_ref = oracle.attention(q, k, v, scale, causal)
        rep = compare(o, lse, o_ref, lse_ref)
    else:
        o_ref, lse_ref = oracle.attention(q, k, v, scale, causal, rows=rows)
        D = q.shape[-1]
        rows_t = torch.as_tensor(rows)
        rep = compare(o.reshape(-1, D)[rows_t], lse.reshape(-1)[rows_t], o_ref, lse_ref)
    assert rep.ok(), str(rep)
    return o, lse, rep


PREFILL_SHAPES = [
    # B, Hq, Hkv, Sq, Skv, D, causal
    (1, 1, 1, 128, 128, 128, True),     # exactly one tile
    (1, 2, 2, 64, 64, 32, True),        # smaller than one tile
    (1, 2, 1, 200, 200, 64, True),      # ragged query and key tails
    (2, 4, 2, 300, 300, 128, True),     # several tiles, ragged tail, GQA 2
    (1, 4, 1, 256, 768, 128, True),     # cache offset 512, GQA 4
    (1, 2, 2, 130, 1000, 128, True),    # offset 870, ragged
    (1, 8, 1, 333, 333, 64, False),     # non-causal, GQA 8
    (1, 2, 2, 2, 2, 128, True),         # smallest prefill
    (1, 2, 2, 5, 1, 64, False),         # non-causal with more queries than keys
    (1, 2, 2, 129, 129, 32, True),      # one row past a tile
    (2, 16, 2, 64, 96, 128, True),      # GQA 8 with a short cache offset
    (1, 3, 3, 100, 300, 64, False),     # non-causal over a longer cache
    (1, 4, 1, 512, 512, 128, True),     # four diagonal tiles
    (1, 1, 1, 1000, 1200, 32, True),    # D 32, offset 200
    (1, 6, 2, 300, 300, 64, True),      # odd GQA group 3: the two tiles of a CTA are consecutive rows
    (2, 8, 4, 257, 257, 128, True),     # GQA 2: the two tiles of a CTA are two heads, one row past
]


@pytest.mark.parametrize("shape", PREFILL_SHAPES, ids=lambda s: "b{}_hq{}_hkv{}_sq{}_skv{}_d{}_{}".format(
    *s[:6], "c" if s[6] else "nc"))
def test_prefill_matches_oracle(shape):
    B, Hq, Hkv, Sq, Skv, D, causal = shape
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, D, causal, seed=sum(shape[:6]))
    q, k, v = inputs.generate(w)
    check(q, k, v, w.scale, causal)


DECODE_SHAPES = [
    # B, Hq, Hkv, Skv, D
    (2, 8, 8, 77, 64),       # group 1, ragged
    (3, 16, 2, 1000, 128),   # group 8
    (1, 6, 1, 300, 32),      # group 6 -> 2 heads per CTA
    (4, 4, 4, 1, 128),       # a single cached key
    (2, 12, 4, 5000, 128),   # group 3 -> 1 head per CTA
    (1, 32, 8, 64, 128),     # exactly one chunk
    (2, 32, 8, 65, 128),     # one key into the second chunk
    (2, 4, 2, 257, 128),     # group 2 on the tensor core, ragged last chunk
    (2, 32, 2, 700, 128),    # group 16: all sixteen MMA columns used
    (1, 64, 2, 300, 128),    # group 32 -> two pairs of 16 heads per kv head
]


@pytest.mark.parametrize("shape", DECODE_SHAPES, ids=lambda s: "b{}_hq{}_hkv{}_skv{}_d{}".format(*s))
def test_decode_matches_oracle(shape):
    B, Hq, Hkv, Skv, D = shape
    w = inputs.custom(B, Hq, Hkv, 1, Skv, D, True, seed=7 * Skv + D)
    q, k, v = inputs.generate(w)
    check(q, k, v, w.scale, True)


@pytest.mark.parametrize("ctas", [1, 2, 3, 7, 16, 61, 64, 97, 500])
def test_decode_cta_count_does_not_matter(ctas):
    """The decode spreads the pairs' key chunks over any number of CTAs (shared pairs are merged
    through their LSEs): the result does not depend on that number beyond rounding."""
    w = inputs.custom(2, 8, 2, 1, 4000, 128, True, seed=99)
    q, k, v = inputs.generate(w)
    o, lse, _ = check(q, k, v, w.scale, True, decode_ctas=ctas)
    o1, lse1 = run_gpu(q, k, v, w.scale, True, decode_ctas=4)  # one CTA per (batch, kv head)
    assert (o.float() - o1.float()).abs().max().item() <= 2 ** -7
    assert (lse - lse1).abs().max().item() <= 1e-4


def test_decode_many_short_caches_share_ctas():
    """More (batch, kv head) pairs than CTAs, each with a short cache: CTAs cover several pairs."""
    w = inputs.custom(64, 16, 4, 1, 37, 64, True, seed=98)
    q, k, v = inputs.generate(w)
    check(q, k, v, w.scale, True)
    check(q, k, v, w.scale, True, decode_ctas=5)


# ------------------------------------------------------------------------------ the five workloads

def test_tiny_prefill_workload_full():
    w = inputs.TINY_PREFILL
    q, k, v = inputs.generate(w)
    check(q, k, v, w.scale, w.causal)


def test_prefill_8b_workload_sampled_rows():
    w = inputs.PREFILL_8B
    q, k, v = inputs.generate(w)
    check(q, k, v, w.scale, w.causal, rows=inputs.sample_rows(w, every=61).numpy())


def test_decode_workload_full():
    w = inputs.DECODE_GQA
    q, k, v = inputs.generate(w)
    check(q, k, v, w.scale, w.causal)


def test_chunked_prefill_workload_full():
    w = inputs.CHUNKED_PREFILL
    q, k, v = inputs.generate(w)
    check(q, k, v, w.scale, w.causal)


@pytest.mark.slow
def test_long_prefill_workload_sampled_rows():
    w = inputs.LONG_PREFILL
    q, k, v = inputs.generate(w)
    check(q, k, v, w.scale, w.causal, rows=inputs.sample_rows(w, every=1021).numpy())


# ------------------------------------------------------------------------------ invariants on the GPU

def test_chunk_equals_tail_of_full_prefill_bitwise():
    """Queries 512..767 over a 768-key cache give the same bits as the last rows of a full causal
    prefill: the mask is aligned to the last Sq key columns."""
    w = inputs.custom(1, 4, 2, 768, 768, 128, True, seed=5)
    q, k, v = inputs.generate(w)
    o_full, l_full = run_gpu(q, k, v, w.scale, True)
    o_c, l_c = run_gpu(q[:, :, 512:].contiguous(), k, v, w.scale, True)
    assert torch.equal(o_full[:, :, 512:], o_c) and torch.equal(l_full[:, :, 512:], l_c)


def test_prefix_rows_unchanged_when_tokens_are_appended():
    w = inputs.custom(1, 2, 1, 1000, 1000, 128, True, seed=6)
    q, k, v = inputs.generate(w)
    o_full, l_full = run_gpu(q, k, v, w.scale, True)
    n = 700
    o_pre, l_pre = run_gpu(q[:, :, :n].contiguous(), k[:, :, :n].contiguous(), v[:, :, :n].contiguous(), w.scale, True)
    full_tiles = (n // 128) * 128  # rows whose whole 128-row tile lies inside the prefix
    assert torch.equal(o_full[:, :, :full_tiles], o_pre[:, :, :full_tiles])
    assert torch.equal(l_full[:, :, :full_tiles], l_pre[:, :, :full_tiles])
    assert (o_full[:, :, :n].float() - o_pre.float()).abs().max().item() <= 2 ** -7
    assert (l_full[:, :, :n] - l_pre).abs().max().item() <= 1e-5


def test_decode_equals_last_row_of_prefill():
    w = inputs.custom(2, 8, 2, 900, 900, 128, True, seed=8)
    q, k, v = inputs.generate(w)
    o_full, l_full = run_gpu(q, k, v, w.scale, True)
    o_d, l_d = run_gpu(q[:, :, -1:].contiguous(), k, v, w.scale, True)
    o_n, l_n = run_gpu(q[:, :, -1:].contiguous(), k, v, w.scale, False)
    assert torch.equal(o_d, o_n) and torch.equal(l_d, l_n)  # decode needs no mask
    assert (o_full[:, :, -1:].float() - o_d.float()).abs().max().item() <= 2 ** -7
    assert (l_full[:, :, -1:] - l_d).abs().max().item() <= 1e-4


def test_zero_query_gives_prefix_mean():
    """q = 0: every visible score is 0, so O_i is the mean of the visible V rows, LSE_i = ln(count)."""
    B, H, Sq, Skv, D = 1, 2, 300, 700, 128
    w = inputs.custom(B, H, H, Sq, Skv, D, True, seed=9)
    _, k, v = inputs.generate(w)
    q = torch.zeros((B, H, Sq, D), dtype=torch.bfloat16)
    o, lse = run_gpu(q, k, v, w.scale, True)
    vd = v.double()
    csum = vd.cumsum(dim=2)
    counts = torch.arange(Skv - Sq + 1, Skv + 1, dtype=torch.float64)
    mean = csum[:, :, Skv - Sq:] / counts.view(1, 1, -1, 1)
    assert (o.double() - mean).abs().max().item() <= 1e-2
    assert (lse.double() - counts.log().view(1, 1, -1)).abs().max().item() <= 1e-3


def test_key_shift_invariance():
    """Adding one vector u to every key adds scale*(q.u) to each score of a row: O is unchanged and
    LSE moves by scale*(q.u). Values are multiples of 1/8 small enough that K + u is exact in bf16."""
    g = torch.Generator().manual_seed(10)
    B, Hq, Hkv, S, D = 1, 4, 2, 400, 128
    q = (torch.randint(-8, 9, (B, Hq, S, D), generator=g) / 8.0).to(torch.bfloat16)
    k = (torch.randint(-64, 65, (B, Hkv, S, D), generator=g) / 8.0).to(torch.bfloat16)
    v = torch.randn((B, Hkv, S, D), generator=g).to(torch.bfloat16)
    u = (torch.randint(-32, 33, (B, Hkv, 1, D), generator=g) / 8.0)
    k2 = (k.double() + u.double()).to(torch.bfloat16)
    assert torch.equal(k2.double(), k.double() + u.double())
    scale = 1.0 / math.sqrt(D)
    o1, l1 = run_gpu(q, k, v, scale, True)
    o2, l2 = run_gpu(q, k2, v, scale, True)
    ur = u.repeat_interleave(Hq // Hkv, dim=1)
    shift = float(np.float32(scale)) * (q.double() * ur.double()).sum(-1)
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l2.double() - l1.double() - shift).abs().max().item() <= 1e-3


def test_inputs_read_and_outputs_written_only_in_bounds():
    """K/V sit inside NaN-filled buffers and O/LSE inside sentinel-filled ones: no NaN may leak in
    (no key past Skv is read) and the sentinels must survive (nothing is written out of bounds)."""
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 2, 200, 333, 128
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, D, True, seed=11)
    q, k, v = inputs.generate(w)
    pad = 4096
    nan = float("nan")
    kbuf = torch.full((2 * pad + k.numel(),), nan, dtype=torch.bfloat16, device="cuda")
    vbuf = torch.full((2 * pad + v.numel(),), nan, dtype=torch.bfloat16, device="cuda")
    kbuf[pad:pad + k.numel()] = k.reshape(-1).cuda()
    vbuf[pad:pad + v.numel()] = v.reshape(-1).cuda()
    obuf = torch.full((2 * pad + q.numel(),), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((2 * pad + B * Hq * Sq,), 7.0, dtype=torch.float32, device="cuda")
    kd = kbuf[pad:pad + k.numel()].view(k.shape)
    vd = vbuf[pad:pad + v.numel()].view(v.shape)
    od = obuf[pad:pad + q.numel()].view(q.shape)
    ld = lbuf[pad:pad + B * Hq * Sq].view(B, Hq, Sq)
    for sq in (Sq, 1):  # prefill and decode
        qd = q[:, :, :sq].contiguous().cuda()
        o_view = obuf[pad:pad + qd.numel()].view(qd.shape)
        l_view = lbuf[pad:pad + B * Hq * sq].view(B, Hq, sq)
        obuf.fill_(7.0)
        lbuf.fill_(7.0)
        attn.attn_fwd(qd, kd, vd, scale=w.scale, causal=True, out=o_view, lse=l_view)
        torch.cuda.synchronize()
        assert torch.isfinite(o_view.float()).all() and torch.isfinite(l_view).all()
        assert (obuf[:pad] == 7.0).all() and (obuf[pad + qd.numel():] == 7.0).all()
        assert (lbuf[:pad] == 7.0).all() and (lbuf[pad + B * Hq * sq:] == 7.0).all()
        o_ref, lse_ref = oracle.attention(q[:, :, :sq].contiguous(), k, v, w.scale, True)
        rep = compare(o_view, l_view, o_ref, lse_ref)
        assert rep.ok(), str(rep)
    del od, ld


def test_binding_rejects_bad_tensors():
    q = torch.zeros((1, 2, 8, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TypeError):
        attn.attn_fwd(q.float(), q, q)
    with pytest.raises(ValueError):
        attn.attn_fwd(q.transpose(2, 3), q, q)
    with pytest.raises(attn.AttnError) as e:
        attn.attn_fwd(q, q[:, :, :4].contiguous(), q[:, :, :4].contiguous(), causal=True)
    assert e.value.status == -6


# ------------------------------------------------------------------------------ scale other than 1/sqrt(D)
# The boundary takes any finite scale > 0 and applies it as given ("05 · Tích vô hướng…", "Vì sao
# chia cho √128" explains 1/sqrt(d) as the usual choice, not the only one). V is multiplied by 1/4
# (exact in bf16) so that |O| < 2: a peaked softmax puts O close to single V rows, and for |O| >= 4
# half a bf16 ulp of the output alone would exceed the 1e-2 bound.

SCALE_SHAPES = [
    # B, Hq, Hkv, Sq, Skv, D, causal
    (1, 4, 2, 300, 300, 128, True),
    (1, 4, 2, 100, 500, 128, True),    # cache offset 400
    (1, 2, 2, 200, 456, 64, False),
    (1, 2, 1, 257, 257, 32, True),
    (2, 8, 2, 1, 777, 128, True),      # decode, tensor core
    (2, 8, 8, 1, 300, 64, True),       # decode, CUDA cores
    (1, 6, 1, 1, 300, 32, True),
]


@pytest.mark.parametrize("scale", [0.05, 0.3, 2.0])
@pytest.mark.parametrize("shape", SCALE_SHAPES, ids=lambda s: "b{}_hq{}_hkv{}_sq{}_skv{}_d{}_{}".format(
    *s[:6], "c" if s[6] else "nc"))
def test_scale_other_than_inverse_sqrt_d(shape, scale):
    B, Hq, Hkv, Sq, Skv, D, causal = shape
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, D, causal, seed=sum(shape[:6]) + int(100 * scale))
    q, k, v = inputs.generate(w)
    v = (v.float() * 0.25).to(torch.bfloat16)
    scale32 = float(np.float32(scale))
    check(q, k, v, scale32, causal)


@pytest.mark.parametrize("shape", [(1, 4, 2, 1024, 1024, 128, True), (4, 32, 8, 1, 4096, 128, True),
                                   (1, 4, 4, 600, 600, 64, True)],
                         ids=["prefill_d128", "decode_d128", "prefill_d64"])
def test_high_variance_scores_drive_the_lazy_rescale(shape):
    """Q and K drawn N(0, 4^2) (the N(0,1) draws times 4, exact in bf16): with scale 1/sqrt(D) the
    scores have a standard deviation of 16, so the running max of ordinary rows jumps past the
    rescale threshold again and again, not only on the 32K workload's outlier keys."""
    B, Hq, Hkv, Sq, Skv, D, causal = shape
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, D, causal, seed=4242 + Sq)
    q, k, v = inputs.generate(w)
    q = (q.float() * 4).to(torch.bfloat16)
    k = (k.float() * 4).to(torch.bfloat16)
    v = (v.float() * 0.25).to(torch.bfloat16)
    check(q, k, v, w.scale, causal)


def test_workspace_growth_does_not_synchronise():
    """A decode that needs a larger workspace than any call before it returns while earlier work on
    its stream is still running: the workspace grows stream-ordered (no device synchronisation)."""
    # Both shapes run the same kernel instantiation (D = 32, one head per kv head), so the first
    # call has loaded it; the second needs 65536 arrival counters, more than any test before it.
    small = inputs.custom(1, 4, 4, 1, 8, 32, True, seed=1)
    big = inputs.custom(16384, 4, 4, 1, 8, 32, True, seed=2)
    qs, ks, vs = (t.cuda() for t in inputs.generate(small))
    qb, kb, vb = (t.cuda() for t in inputs.generate(big))
    ob = torch.empty_like(qb)
    lb = torch.empty(qb.shape[:3], dtype=torch.float32, device="cuda")
    attn.attn_fwd(qs, ks, vs, scale=small.scale)  # loads the kernels and creates the workspace
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    done = torch.cuda.Event()
    torch.cuda._sleep(2_000_000_000)  # about one second of device time
    done.record(stream)
    attn.attn_fwd(qb, kb, vb, scale=big.scale, out=ob, lse=lb)  # grows the workspace
    still_running = not done.query()
    torch.cuda.synchronize()
    assert still_running, "attn_fwd waited for earlier work while growing its workspace"
    o_ref, lse_ref = oracle.attention(qb.cpu(), kb.cpu(), vb.cpu(), big.scale, True)
    rep = compare(ob, lb, o_ref, lse_ref)
    assert rep.ok(), str(rep)


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2, reason="needs two devices")
def test_second_device_gets_its_own_kernel_attributes():
    """Function attributes (the dynamic shared-memory limit) are set per device: a prefill and a
    decode on a second device run after the first device has used both."""
    w = inputs.custom(1, 4, 2, 300, 300, 128, True, seed=12)
    q, k, v = inputs.generate(w)
    for dev in (0, 1):
        with torch.cuda.device(dev):
            o, lse = attn.attn_fwd(q.to(dev), k.to(dev), v.to(dev), scale=w.scale, causal=True)
            od, ld = attn.attn_fwd(q[:, :, -1:].contiguous().to(dev), k.to(dev), v.to(dev), scale=w.scale)
            torch.cuda.synchronize(dev)
        o_ref, lse_ref = oracle.attention(q, k, v, w.scale, True)
        assert compare(o, lse, o_ref, lse_ref).ok()
