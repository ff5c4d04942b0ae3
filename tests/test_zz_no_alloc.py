"""attn_decode_noalloc: the decode entry point that allocates nothing, for callers that must not
have the library call cudaMalloc (a latency-bound serving loop that cannot take the device
synchronisation of an allocation mid-request, or a process whose device memory belongs to one
allocator or a budget fixed at start-up). Its scratch is a fixed array in the library's device
memory. These tests call it through the C ABI and compare it with attn_fwd and with the fp64
oracle, within the parity tolerance, on two calls in a row: the second call must not be disturbed
by what the first left in the shared array. After its first call on a device (which looks up the
array's address and, with CUDA's lazy module loading, makes the runtime load the array), a call
must leave the device's free memory unchanged. This file is collected last so that a run stopping
at the first failure has run every other test before it."""
import ctypes

import pytest
import torch

import oracle
from causal_attention_attn_b200 import attn, build, inputs
from tests.compare import compare

pytestmark = pytest.mark.gpu

O_MAX_ABS, O_MEAN_ABS, LSE_MAX_ABS = 1e-2, 1e-3, 1e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available() or torch.cuda.get_device_capability(0) != (10, 0):
        pytest.skip("needs an sm_100 device")
    build.build()
    return attn.load_library()


def call_noalloc(lib, q, k, v, o, lse, scale):
    B, Hq, _, D = q.shape
    _, Hkv, Skv, _ = k.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.attn_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   B, Hq, Hkv, Skv, D, ctypes.c_float(scale), stream)


def assert_close(o, lse, o_ref, lse_ref):
    err = (o.float() - o_ref.float()).abs()
    assert err.max().item() <= O_MAX_ABS and err.mean().item() <= O_MEAN_ABS, (err.max().item(), err.mean().item())
    assert (lse - lse_ref).abs().max().item() <= LSE_MAX_ABS


@pytest.mark.parametrize("shape", [(16, 32, 8, 4096, 128), (3, 12, 4, 777, 64), (2, 8, 8, 65, 32)],
                         ids=lambda s: "b{}_hq{}_hkv{}_skv{}_d{}".format(*s))
def test_matches_attn_fwd_and_oracle_on_two_calls_in_a_row(lib, shape):
    B, Hq, Hkv, Skv, D = shape
    for call in range(2):
        w = inputs.custom(B, Hq, Hkv, 1, Skv, D, True, seed=1000 * call + Skv)
        qh, kh, vh = inputs.generate(w)
        q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
        o_ref, lse_ref = attn.attn_fwd(q, k, v, scale=w.scale, causal=True)
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, Hq, 1), float("nan"), dtype=torch.float32, device="cuda")
        rc = call_noalloc(lib, q, k, v, o, lse, w.scale)
        torch.cuda.synchronize()
        assert rc == 0, attn.status_string(rc)
        assert_close(o, lse, o_ref, lse_ref)
        o64, lse64 = oracle.attention(qh, kh, vh, w.scale, True)
        rep = compare(o, lse, o64, lse64)
        assert rep.ok(), f"call {call}: {rep}"
    assert attn.device_status() == 0


def test_second_call_leaves_free_device_memory_unchanged(lib):
    w = inputs.custom(4, 32, 8, 1, 2048, 128, True, seed=31)
    q, k, v = (t.cuda() for t in inputs.generate(w))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, 1), dtype=torch.float32, device="cuda")
    assert call_noalloc(lib, q, k, v, o, lse, w.scale) == 0  # first call on this device: set-up
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        assert call_noalloc(lib, q, k, v, o, lse, w.scale) == 0
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, (free_before, free_after)


def test_rejects_problems_beyond_the_scratch_limit(lib):
    # 2.2 million (batch, kv head) pairs need 8.8 MB of counters, more than the 8 MiB array. The
    # tensors are real and sized for the shape, so nothing here could read out of bounds.
    B, Hq, Hkv, Skv, D = 2_200_000, 1, 1, 1, 32
    q = torch.zeros((B, Hq, 1, D), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, Hkv, Skv, D), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
    rc = call_noalloc(lib, q, k, k, o, lse, 0.5)
    torch.cuda.synchronize()
    assert rc == -13, rc
    assert "scratch" in attn.status_string(rc)
