"""GPU tests of attn_fwd_host: host buffers in and out, the copies pipelined against the attention
slice by slice. Prefill results must equal attn_fwd's bit for bit (every (batch, head) problem is
computed the same way whatever the slicing); the decode (whose split over CTAs depends on the
problem count) is checked against the fp64 oracle. Tolerance (tests/compare.py): O max|err| <= 1e-2,
mean|err| <= 1e-3; LSE max|err| <= 1e-3.
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
    assert attn.device_status() == 0, "a kernel-side wait ran out during the host-buffer tests"


SHAPES = [
    # B, Hq, Hkv, Sq, Skv, D, causal
    (1, 32, 8, 1024, 1024, 128, True),   # eight units: halves of the first and last, one per slice between
    (3, 6, 3, 130, 400, 128, True),      # nine units over eight slices; group * Sq even
    (2, 5, 5, 67, 67, 64, True),         # ten units; group * Sq odd: slices fall on whole lse blocks
    (1, 4, 1, 257, 300, 32, False),      # one unit
    (16, 32, 8, 200, 600, 128, True),    # 128 units; the first and last in halves of their heads
    (2, 4, 2, 256, 300, 128, True),      # four units; halves of one head each at both ends
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b{}_hq{}_hkv{}_sq{}_skv{}_d{}_{}".format(
    *s[:6], "c" if s[6] else "nc"))
def test_host_call_equals_attn_fwd_bitwise(shape):
    B, Hq, Hkv, Sq, Skv, D, causal = shape
    w = inputs.custom(B, Hq, Hkv, Sq, Skv, D, causal, seed=sum(shape[:6]))
    q, k, v = inputs.generate(w)
    o_ref, l_ref = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=w.scale, causal=causal)
    o, lse = attn.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), scale=w.scale, causal=causal)
    assert torch.equal(o, o_ref.cpu()) and torch.equal(lse, l_ref.cpu())


def test_host_decode_matches_oracle():
    w = inputs.custom(16, 32, 8, 1, 2000, 128, True, seed=5)
    q, k, v = inputs.generate(w)
    o, lse = attn.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), scale=w.scale, causal=True)
    rep = compare(o, lse, *oracle.attention(q, k, v, w.scale, True))
    assert rep.ok(), str(rep)


def test_pageable_host_memory_gives_the_same_result():
    w = inputs.custom(2, 8, 2, 300, 300, 128, True, seed=8)
    q, k, v = inputs.generate(w)
    o_pin, l_pin = attn.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), scale=w.scale)
    o, lse = attn.attn_fwd_host(q.clone(), k.clone(), v.clone(), scale=w.scale,
                                out_host=torch.empty_like(o_pin), lse_host=torch.empty_like(l_pin))
    assert torch.equal(o, o_pin) and torch.equal(lse, l_pin)


def test_copies_wait_for_earlier_work_on_the_stream_and_stay_in_bounds():
    """Device staging buffers still being written by earlier work on the stream are copied over only
    after it; the host outputs sit inside sentinel-filled buffers that must survive."""
    w = inputs.custom(3, 6, 3, 130, 400, 128, True, seed=11)
    q, k, v = inputs.generate(w)
    o_ref, l_ref = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=w.scale, causal=True)
    stream = torch.cuda.Stream()
    dev = (torch.empty(q.shape, dtype=torch.bfloat16, device="cuda"),
           torch.empty(k.shape, dtype=torch.bfloat16, device="cuda"),
           torch.empty(v.shape, dtype=torch.bfloat16, device="cuda"),
           torch.empty(q.shape, dtype=torch.bfloat16, device="cuda"),
           torch.empty(q.shape[:3], dtype=torch.float32, device="cuda"))
    pad = 4096
    obuf = torch.full((2 * pad + q.numel(),), 7.0, dtype=torch.bfloat16).pin_memory()
    lbuf = torch.full((2 * pad + q.numel() // q.shape[3],), 7.0, dtype=torch.float32).pin_memory()
    o_host = obuf[pad:pad + q.numel()].view(q.shape)
    l_host = lbuf[pad:pad + q.numel() // q.shape[3]].view(q.shape[:3])
    with torch.cuda.stream(stream):
        torch.cuda._sleep(50_000_000)  # earlier work on the stream ...
        for t in dev:
            t.fill_(float("nan"))       # ... that writes the staging buffers last
    o, lse = attn.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), scale=w.scale, stream=stream,
                                out_host=o_host, lse_host=l_host, dev_bufs=dev)
    assert torch.equal(o, o_ref.cpu()) and torch.equal(lse, l_ref.cpu())
    assert (obuf[:pad] == 7.0).all() and (obuf[pad + q.numel():] == 7.0).all()
    assert (lbuf[:pad] == 7.0).all() and (lbuf[pad + q.numel() // q.shape[3]:] == 7.0).all()


def test_concurrent_host_calls_from_two_threads():
    """Two host threads calling at once on their own streams (the library's copy streams and events
    are shared, so the calls queue one after another): each gets its own, correct result."""
    import threading

    shapes = [inputs.custom(2, 8, 2, 200, 333, 128, True, seed=101), inputs.custom(1, 4, 4, 130, 600, 64, True, seed=102)]
    data = [tuple(t.pin_memory() for t in inputs.generate(w)) for w in shapes]
    refs = [attn.attn_fwd(*(t.cuda() for t in d), scale=w.scale, causal=True) for w, d in zip(shapes, data)]
    torch.cuda.synchronize()
    results, errors = [None, None], []

    def worker(i):
        try:
            torch.cuda.set_device(0)
            stream = torch.cuda.Stream()
            outs = []
            for _ in range(5):
                outs.append(attn.attn_fwd_host(*data[i], scale=shapes[i].scale, causal=True, stream=stream))
            results[i] = outs
        except Exception as e:  # reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for i in range(2):
        for o, lse in results[i]:
            assert torch.equal(o, refs[i][0].cpu()) and torch.equal(lse, refs[i][1].cpu()), i
