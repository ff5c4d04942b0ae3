"""GPU parity of the LSE merge kernel (``attn_lse_merge``) and of ring attention's per-block work.

Every run here has one GPU, so no test waits on another rank: the ring's schedule is emulated on
one GPU (the chunks are indexed instead of received), which runs exactly the kernels and the
merge order a rank runs; the distributed ring loop itself is run with one rank, and with two and
three gloo ranks on the CPU in ``test_ring_cpu.py``.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from causal_attention_attn_b200 import attn, build, inputs
from causal_attention_attn_b200.ring import DIAG, ring_schedule, zigzag_shard
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
    assert attn.device_status() == 0, "a kernel-side wait ran out during the ring tests"


@pytest.mark.parametrize("D", [32, 64, 128])
def test_merge_of_two_key_blocks_equals_attention_over_both(D):
    """Attention over keys [0, h) and over [h, Skv), merged, equals attention over all keys."""
    w = inputs.custom(2, 4, 2, 96, 200, D, False, seed=D)
    q, k, v = inputs.generate(w)
    h = 77
    parts = [oracle.attention(q, k[:, :, :h].contiguous(), v[:, :, :h].contiguous(), w.scale, False),
             oracle.attention(q, k[:, :, h:].contiguous(), v[:, :, h:].contiguous(), w.scale, False)]
    o_acc = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    lse_acc = torch.full(q.shape[:-1], float("-inf"), dtype=torch.float32, device="cuda")
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    for n, (o_p, l_p) in enumerate(parts):
        attn.attn_lse_merge(o_acc, lse_acc, torch.from_numpy(o_p).to(torch.bfloat16).cuda(),
                            torch.from_numpy(l_p).float().cuda(), out=out if n == 1 else None)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(q, k, v, w.scale, False)
    rep = compare(out, lse_acc, ro, rl)
    assert rep.ok(), str(rep)


def test_merge_with_empty_sides():
    """lse = -inf means no key: such a side has weight 0; a row empty on both sides stays empty."""
    rows, D = 40, 128
    g = torch.Generator().manual_seed(1)
    o_a = torch.randn((rows, D), generator=g)
    l_a = torch.randn((rows,), generator=g)
    o_p = torch.randn((rows, D), generator=g).to(torch.bfloat16)
    l_p = torch.randn((rows,), generator=g)
    l_a[:10] = float("-inf")
    o_a[:10] = 0.0
    l_p[10:20] = float("-inf")
    l_a[20:30] = float("-inf")
    l_p[20:30] = float("-inf")
    o_a[20:30] = 0.0
    acc, lacc = o_a.clone().cuda(), l_a.clone().cuda()
    attn.attn_lse_merge(acc, lacc, o_p.cuda(), l_p.cuda())
    torch.cuda.synchronize()
    acc, lacc = acc.cpu(), lacc.cpu()
    assert torch.equal(acc[:10], o_p[:10].float()) and torch.equal(lacc[:10], l_p[:10])   # empty accumulator
    assert torch.equal(acc[10:20], o_a[10:20]) and torch.equal(lacc[10:20], l_a[10:20])   # empty part
    assert torch.equal(acc[20:30], o_a[20:30]) and bool(torch.isneginf(lacc[20:30]).all())  # both empty
    m = torch.maximum(l_a[30:], l_p[30:]).double()
    wa, wp = torch.exp(l_a[30:].double() - m), torch.exp(l_p[30:].double() - m)
    want = (wa[:, None] * o_a[30:].double() + wp[:, None] * o_p[30:].double()) / (wa + wp)[:, None]
    assert torch.allclose(acc[30:].double(), want, rtol=1e-5, atol=1e-5)
    assert torch.allclose(lacc[30:].double(), m + torch.log(wa + wp), rtol=0, atol=1e-5)


@pytest.mark.parametrize("world,S,causal", [(4, 128, True), (3, 100, True), (2, 64, False)])
def test_ring_schedule_on_one_gpu_matches_oracle(world, S, causal):
    """Every virtual rank runs its zigzag schedule's blocks through attn_fwd and attn_lse_merge.
    S: tokens per rank (two chunks of S / 2)."""
    w = inputs.custom(1, 8, 2, world * S, world * S, 128, causal, seed=world * S)
    q, k, v = (t.cuda() for t in inputs.generate(w))
    ro, rl = oracle.attention(*(t.cpu() for t in (q, k, v)), w.scale, causal)
    c = S // 2

    def halves(x):
        return x[:, :, :c].contiguous(), x[:, :, c:].contiguous()

    for rank in range(world):
        qs = halves(zigzag_shard(q, rank, world))
        o_acc = [torch.zeros(x.shape, dtype=torch.float32, device="cuda") for x in qs]
        lse_acc = [torch.full(x.shape[:-1], float("-inf"), dtype=torch.float32, device="cuda") for x in qs]
        out = [torch.empty(x.shape, dtype=torch.bfloat16, device="cuda") for x in qs]
        sched = ring_schedule(rank, world, causal)
        last = {qh: (t, b) for t, _, blocks in sched for b, (qh, _, _) in enumerate(blocks)}
        for t, j, blocks in sched:
            ks, vs = halves(zigzag_shard(k, j, world)), halves(zigzag_shard(v, j, world))
            for b, (qh, kh, mode) in enumerate(blocks):
                o_p, l_p = attn.attn_fwd(qs[qh], ks[kh], vs[kh], scale=w.scale, causal=(mode == DIAG))
                attn.attn_lse_merge(o_acc[qh], lse_acc[qh], o_p, l_p, out=out[qh] if last[qh] == (t, b) else None)
        torch.cuda.synchronize()
        want_o = zigzag_shard(torch.from_numpy(ro), rank, world).numpy()
        want_l = zigzag_shard(torch.from_numpy(rl), rank, world).numpy()
        rep = compare(torch.cat(out, dim=2), torch.cat(lse_acc, dim=2), want_o, want_l)
        assert rep.ok(), f"rank {rank}: {rep}"


def test_ring_loop_with_one_rank_equals_attn_fwd():
    import torch.distributed as dist

    from causal_attention_attn_b200.ring import ring_attention

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        w = inputs.custom(1, 4, 2, 200, 200, 128, True, seed=4)
        q, k, v = (t.cuda() for t in inputs.generate(w))
        o, lse = ring_attention(q, k, v, scale=w.scale, causal=True)
        ro, rl = oracle.attention(*(t.cpu() for t in (q, k, v)), w.scale, True)
        rep = compare(o, lse, ro, rl)
        assert rep.ok(), str(rep)
    finally:
        dist.destroy_process_group()


def test_merge_reproduces_the_pages_online_softmax_example():
    """The blocks [2, 1] and [3, 0] of the worked online-softmax example ("05 · Tích vô hướng,
    Softmax và toán của Attention", §6), with one-hot value rows so that O is the weight vector:
    the partial LSEs ln(e^2 + e) and ln(e^3 + 1) merge to ln(e^2 + e + e^3 + 1) = 3.440190 and O to
    softmax(2, 1, 3, 0)."""
    import json
    import math

    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pages_worked_examples.json")) as f:
        blocks = json.load(f)["online_softmax_blocks"]["blocks"]
    D = 32

    def partial(scores, first_key):
        lse = math.log(sum(math.exp(s) for s in scores))
        o = torch.zeros(D)
        for n, s in enumerate(scores):
            o[first_key + n] = math.exp(s - lse)  # value row of key j is the unit vector e_j
        return o.to(torch.bfloat16), lse

    (o1, l1), (o2, l2) = partial(blocks[0], 0), partial(blocks[1], len(blocks[0]))
    o_acc = o1.float().reshape(1, D).cuda()
    lse_acc = torch.tensor([l1], dtype=torch.float32, device="cuda")
    out = torch.empty((1, D), dtype=torch.bfloat16, device="cuda")
    attn.attn_lse_merge(o_acc, lse_acc, o2.reshape(1, D).cuda(), torch.tensor([l2], dtype=torch.float32, device="cuda"),
                        out=out)
    torch.cuda.synchronize()
    scores = blocks[0] + blocks[1]
    want_lse = math.log(sum(math.exp(s) for s in scores))
    assert abs(want_lse - 3.440190) < 1e-6
    assert abs(lse_acc.item() - want_lse) < 1e-5
    want = [math.exp(s - want_lse) for s in scores]
    got = out.float().cpu()[0]
    for j, wj in enumerate(want):
        assert abs(got[j].item() - wj) <= 5e-3 * wj, (j, got[j].item(), wj)  # two bf16 roundings: <= 2^-8
    assert torch.all(got[len(scores):] == 0)


def test_merge_reads_and_writes_only_in_bounds():
    """The part inside NaN-filled buffers, the accumulator and the output inside sentinel-filled
    ones: the sentinels must survive and no NaN may leak into the merged rows."""
    rows, D, pad = 37, 128, 4096
    g = torch.Generator().manual_seed(2)
    o_a, l_a = torch.randn((rows, D), generator=g), torch.randn((rows,), generator=g)
    o_p, l_p = torch.randn((rows, D), generator=g).to(torch.bfloat16), torch.randn((rows,), generator=g)

    def inside(t, fill):
        buf = torch.full((2 * pad + t.numel(),), fill, dtype=t.dtype, device="cuda")
        buf[pad:pad + t.numel()] = t.reshape(-1).cuda()
        return buf, buf[pad:pad + t.numel()].view(t.shape)

    abuf, acc = inside(o_a, 7.0)
    lbuf, lacc = inside(l_a, 7.0)
    _, part = inside(o_p, float("nan"))
    _, lpart = inside(l_p, float("nan"))
    obuf, out = inside(torch.full((rows, D), 7.0, dtype=torch.bfloat16), 7.0)
    attn.attn_lse_merge(acc, lacc, part, lpart, out=out)
    torch.cuda.synchronize()
    for buf, n in ((abuf, rows * D), (lbuf, rows), (obuf, rows * D)):
        assert (buf[:pad] == 7.0).all() and (buf[pad + n:] == 7.0).all()
    assert torch.isfinite(acc).all() and torch.isfinite(lacc).all() and torch.isfinite(out.float()).all()
    m = torch.maximum(l_a, l_p).double()
    wa, wp = torch.exp(l_a.double() - m), torch.exp(l_p.double() - m)
    want = (wa[:, None] * o_a.double() + wp[:, None] * o_p.double()) / (wa + wp)[:, None]
    assert torch.allclose(acc.cpu().double(), want, rtol=1e-5, atol=1e-5)
    assert torch.allclose(out.cpu().double(), want, rtol=2.0 ** -8, atol=1e-6)
