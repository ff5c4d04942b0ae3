"""The C-ABI library loads and exports every entry point include/attn.h declares; argument errors
are reported on the host before anything is launched. No test here needs a GPU: every call either
queries static information or passes arguments the library rejects before touching the device."""
import os
import re

import pytest

from causal_attention_attn_b200 import attn, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return attn.load_library()


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    assert set(declared_functions()) == set(attn.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    syms = os.popen(f"nm -D --defined-only {attn.library_path}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", syms), name


def test_version_and_status_strings(lib):
    assert lib.attn_version() == 700
    for code, name in attn.STATUS_NAMES.items():
        s = attn.status_string(code)
        assert s and s != "unknown status", (code, name)
    assert attn.status_string(12345) == "unknown status"


def test_library_has_no_dynamic_cuda_dependency():
    deps = os.popen(f"ldd {attn.library_path}").read()
    assert "libcuda.so" not in deps and "libcudart.so" not in deps, deps


# Fake, 16-byte-aligned addresses: every case below is rejected before any CUDA call.
A = [0x10000, 0x20000, 0x30000, 0x40000, 0x50000]
GOOD = dict(B=1, Hq=4, Hkv=2, Sq=8, Skv=8, D=64, scale=0.125, causal=1)

CASES = [
    ("null q", dict(ptrs=[0, A[1], A[2], A[3], A[4]]), -1),
    ("null lse", dict(ptrs=[A[0], A[1], A[2], A[3], 0]), -1),
    ("zero batch", dict(B=0), -2),
    ("zero heads", dict(Hq=0), -2),
    ("zero kv heads", dict(Hkv=0), -2),
    ("zero queries", dict(Sq=0), -2),
    ("zero keys", dict(Skv=0), -2),
    ("negative size", dict(Skv=-5), -2),
    ("causal flag 2", dict(causal=2), -2),
    ("rows overflow int32", dict(B=1 << 16, Hq=1 << 8, Hkv=1 << 8, Sq=1 << 8), -2),
    ("gqa not divisible", dict(Hq=6, Hkv=4), -3),
    ("head dim 48", dict(D=48), -4),
    ("head dim 256", dict(D=256), -4),
    ("misaligned k", dict(ptrs=[A[0], A[1] + 8, A[2], A[3], A[4]]), -5),
    ("misaligned o", dict(ptrs=[A[0], A[1], A[2], A[3] + 2, A[4]]), -5),
    ("causal with Sq > Skv", dict(Sq=9, Skv=8), -6),
    ("zero scale", dict(scale=0.0), -11),
    ("negative scale", dict(scale=-0.1), -11),
    ("infinite scale", dict(scale=float("inf")), -11),
    ("nan scale", dict(scale=float("nan")), -11),
]


@pytest.mark.parametrize("name,override,expected", CASES, ids=[c[0] for c in CASES])
def test_argument_errors(lib, name, override, expected):
    args = dict(GOOD)
    args.update({k: v for k, v in override.items() if k != "ptrs"})
    ptrs = override.get("ptrs", A)
    rc = attn.attn_fwd_raw(*ptrs, args["B"], args["Hq"], args["Hkv"], args["Sq"], args["Skv"], args["D"],
                           args["scale"], args["causal"], 0)
    assert rc == expected, (name, rc)


def test_negative_cta_request_rejected(lib):
    rc = lib.attn_fwd_ex(*A, 1, 4, 2, 1, 8, 64, 0.125, 1, -1, None)
    assert rc == -2


def test_non_causal_allows_more_queries_than_keys_in_validation(lib):
    # Validation passes, so the call proceeds to the device query; without a GPU that fails with a
    # CUDA error (or, on a non-sm_100 GPU, an arch error) and still launches nothing.
    import torch

    if torch.cuda.is_available():
        pytest.skip("would reach the device with fake pointers")
    rc = attn.attn_fwd_raw(*A, 1, 4, 2, 9, 8, 64, 0.125, 0, 0)
    assert rc in (-12, -7), rc


PAGED_GOOD = dict(B=2, Hq=8, Hkv=2, num_pages=4, page_size=64, pages_per_seq=2, max_seq_len=128, scale=0.1, ctas=0)
PAGED_CASES = [
    ("null block table", dict(ptrs=[A[0], A[1], A[2], 0, A[4], A[3], A[4]]), -1),
    ("page size 48", dict(page_size=48), -2),
    ("page size 192", dict(page_size=192), -2),
    ("batch 1025", dict(B=1025), -2),
    ("negative max length", dict(max_seq_len=-1), -2),
    ("negative cta count", dict(ctas=-1), -2),
    ("gqa not divisible", dict(Hq=6, Hkv=4), -3),
    ("misaligned seq_lens", dict(ptrs=[A[0], A[1], A[2], A[3], A[4] + 2, A[3], A[4]]), -5),
    ("zero scale", dict(scale=0.0), -11),
]


@pytest.mark.parametrize("name,override,expected", PAGED_CASES, ids=[c[0] for c in PAGED_CASES])
def test_paged_argument_errors(lib, name, override, expected):
    a = dict(PAGED_GOOD)
    a.update({k: v for k, v in override.items() if k != "ptrs"})
    ptrs = override.get("ptrs", [A[0], A[1], A[2], A[3], A[4], A[3], A[4]])
    rc = lib.attn_decode_paged(*ptrs, a["B"], a["Hq"], a["Hkv"], a["num_pages"], a["page_size"], a["pages_per_seq"],
                               a["max_seq_len"], a["scale"], a["ctas"], None)
    assert rc == expected, (name, rc)



# attn_decode_fp8(q, k8, v8, k_scale, v_scale, o, lse, B, Hq, Hkv, Skv, D, scale, ctas, stream)
FP8_GOOD = dict(B=2, Hq=8, Hkv=2, Skv=300, D=128, scale=0.1, ctas=0)
FP8_PTRS = [A[0], A[1], A[2], A[3], A[4], A[0] + 0x100000, A[1] + 0x100000]
FP8_CASES = [
    ("null k_scale", dict(ptrs=FP8_PTRS[:3] + [0] + FP8_PTRS[4:]), -1),
    ("null v_scale", dict(ptrs=FP8_PTRS[:4] + [0] + FP8_PTRS[5:]), -1),
    ("zero keys", dict(Skv=0), -2),
    ("negative cta count", dict(ctas=-1), -2),
    ("gqa not divisible", dict(Hq=6, Hkv=4), -3),
    ("head dim 64", dict(D=64), -4),
    ("misaligned k_scale", dict(ptrs=FP8_PTRS[:3] + [A[3] + 4] + FP8_PTRS[4:]), -5),
    ("misaligned k8", dict(ptrs=[A[0], A[1] + 8] + FP8_PTRS[2:]), -5),
    ("zero scale", dict(scale=0.0), -11),
]


@pytest.mark.parametrize("name,override,expected", FP8_CASES, ids=[c[0] for c in FP8_CASES])
def test_fp8_argument_errors(lib, name, override, expected):
    a = dict(FP8_GOOD)
    a.update({k: v for k, v in override.items() if k != "ptrs"})
    ptrs = override.get("ptrs", FP8_PTRS)
    rc = lib.attn_decode_fp8(*ptrs, a["B"], a["Hq"], a["Hkv"], a["Skv"], a["D"], a["scale"], a["ctas"], None)
    assert rc == expected, (name, rc)


def test_paged_fp8_argument_errors(lib):
    # q, k_pages, v_pages, k_scale, v_scale, block_table, seq_lens, o, lse
    ptrs = [A[0], A[1], A[2], A[3], A[4], A[3], A[4], A[0] + 0x100000, A[1] + 0x100000]
    args = (2, 8, 2, 4, 64, 2, 128, 0.1, 0, None)
    bad_scale = list(ptrs)
    bad_scale[3] = 0
    assert lib.attn_decode_paged_fp8(*bad_scale, *args) == -1
    bad_scale[3] = A[3] + 4
    assert lib.attn_decode_paged_fp8(*bad_scale, *args) == -5
    assert lib.attn_decode_paged_fp8(*ptrs, 2, 8, 2, 4, 48, 2, 128, 0.1, 0, None) == -2


# attn_lse_merge(o_acc, lse_acc, o_part, lse_part, o_out, rows, D, stream)
MERGE_CASES = [
    ("null accumulator", [0, A[1], A[2], A[3], None], 10, 128, -1),
    ("null part lse", [A[0], A[1], A[2], 0, None], 10, 128, -1),
    ("negative rows", [A[0], A[1], A[2], A[3], None], -1, 128, -2),
    ("head dim 48", [A[0], A[1], A[2], A[3], None], 10, 48, -4),
    ("misaligned part", [A[0], A[1], A[2] + 2, A[3], None], 10, 64, -5),
    ("misaligned output", [A[0], A[1], A[2], A[3], A[4] + 8], 10, 32, -5),
    ("no rows: nothing to do", [A[0], A[1], A[2], A[3], None], 0, 128, 0),
]


@pytest.mark.parametrize("name,ptrs,rows,D,expected", MERGE_CASES, ids=[c[0] for c in MERGE_CASES])
def test_lse_merge_argument_errors(lib, name, ptrs, rows, D, expected):
    assert lib.attn_lse_merge(*ptrs, rows, D, None) == expected, name


# attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Sq, Skv, D, scale, causal, stream)
BWD_PTRS = [A[0], A[1], A[2], A[3], A[4], A[0] + 0x100000, A[1] + 0x100000, A[2] + 0x100000, A[3] + 0x100000]
BWD_GOOD = (1, 4, 2, 128, 128, 128, 0.1, 1)
BWD_CASES = [
    ("null dout", 4, 0, BWD_GOOD, -1),
    ("null dv", 8, 0, BWD_GOOD, -1),
    ("null q", 0, 0, BWD_GOOD, -1),
    ("head dim 64", None, None, (1, 4, 2, 128, 128, 64, 0.1, 1), -4),
    ("gqa not divisible", None, None, (1, 6, 4, 128, 128, 128, 0.1, 1), -3),
    ("causal with Sq > Skv", None, None, (1, 4, 2, 129, 128, 128, 0.1, 1), -6),
    ("misaligned dq", 6, A[1] + 0x100000 + 4, BWD_GOOD, -5),
    ("zero scale", None, None, (1, 4, 2, 128, 128, 128, 0.0, 1), -11),
]


@pytest.mark.parametrize("name,slot,value,args,expected", BWD_CASES, ids=[c[0] for c in BWD_CASES])
def test_bwd_argument_errors(lib, name, slot, value, args, expected):
    ptrs = list(BWD_PTRS)
    if slot is not None:
        ptrs[slot] = value
    assert lib.attn_bwd(*ptrs, *args, None) == expected, name


def _strided_call(lib, strides, D=64, B=1, Hq=4, Hkv=2, Sq=8, Skv=8):
    import ctypes

    arrs = [None if s is None else (ctypes.c_longlong * 3)(*s) for s in strides]
    return lib.attn_fwd_strided(A[0], A[1], A[2], A[3], A[4], B, Hq, Hkv, Sq, Skv, D, *arrs, 0.125, 1, None)


@pytest.mark.parametrize("name,strides,D,expected", [
    ("null q strides", [None, (512, 64, 256), (512, 64, 256), (512, 64, 256)], 64, -1),
    ("null o strides", [(512, 64, 256)] * 3 + [None], 64, -1),
    ("stride not a multiple of 8", [(512, 64, 260)] + [(512, 64, 256)] * 3, 64, -5),
    ("zero stride", [(512, 0, 256)] + [(512, 64, 256)] * 3, 64, -5),
    ("negative stride", [(512, 64, 256)] * 3 + [(-512, 64, 256)], 64, -5),
    ("huge stride", [(1 << 40, 64, 256)] + [(512, 64, 256)] * 3, 64, -5),
    ("valid strides, bad head dim", [(512, 64, 256)] * 4, 48, -4),
])
def test_strided_argument_errors(lib, name, strides, D, expected):
    assert _strided_call(lib, strides, D=D) == expected, name


def _prefill_paged_call(lib, **kw):
    a = dict(ptrs=[A[0], A[1], A[2], 0x60000, 0x70000, A[3], A[4]], B=2, Hq=8, Hkv=2, Sq=64, num_pages=10,
             page_size=64, pages_per_seq=4, max_seq_len=256, scale=0.1, causal=1)
    a.update(kw)
    return lib.attn_prefill_paged(*a["ptrs"], a["B"], a["Hq"], a["Hkv"], a["Sq"], a["num_pages"], a["page_size"],
                                  a["pages_per_seq"], a["max_seq_len"], a["scale"], a["causal"], None)


@pytest.mark.parametrize("name,override,expected", [
    ("null seq_lens", dict(ptrs=[A[0], A[1], A[2], 0x60000, 0, A[3], A[4]]), -1),
    ("null o", dict(ptrs=[A[0], A[1], A[2], 0x60000, 0x70000, 0, A[4]]), -1),
    ("zero queries", dict(Sq=0), -2),
    ("page size 48", dict(page_size=48), -2),
    ("page size 192", dict(page_size=192), -2),
    ("negative max_seq_len", dict(max_seq_len=-1), -2),
    ("causal 2", dict(causal=2), -2),
    ("gqa", dict(Hkv=3), -3),
    ("unaligned q", dict(ptrs=[A[0] + 8, A[1], A[2], 0x60000, 0x70000, A[3], A[4]]), -5),
    ("unaligned table", dict(ptrs=[A[0], A[1], A[2], 0x60002, 0x70000, A[3], A[4]]), -5),
    ("zero scale", dict(scale=0.0), -11),
])
def test_prefill_paged_argument_errors(lib, name, override, expected):
    assert _prefill_paged_call(lib, **override) == expected, name


# attn_fwd_host: host pointers are checked first, then the device buffers as attn_fwd checks its
# arguments; every case below is rejected before any CUDA call.
H = [0x110000, 0x120000, 0x130000, 0x140000, 0x150000]


def _fwd_host_call(lib, host=None, dev=None, **kw):
    a = dict(GOOD, **kw)
    host = H if host is None else host
    dev = A if dev is None else dev
    return lib.attn_fwd_host(*host, *dev, a["B"], a["Hq"], a["Hkv"], a["Sq"], a["Skv"], a["D"], a["scale"],
                             a["causal"], None)


FWD_HOST_CASES = [
    ("null q_host", dict(host=[0, H[1], H[2], H[3], H[4]]), -1),
    ("null lse_host", dict(host=[H[0], H[1], H[2], H[3], 0]), -1),
    ("null o_dev", dict(dev=[A[0], A[1], A[2], 0, A[4]]), -1),
    ("misaligned k_dev", dict(dev=[A[0], A[1] + 8, A[2], A[3], A[4]]), -5),
    ("group not integral", dict(Hq=3, Hkv=2), -3),
    ("head dim 48", dict(D=48), -4),
    ("causal with Sq > Skv", dict(Sq=9, Skv=8), -6),
    ("zero scale", dict(scale=0.0), -11),
]


@pytest.mark.parametrize("name,override,expected", FWD_HOST_CASES, ids=[c[0] for c in FWD_HOST_CASES])
def test_fwd_host_argument_errors(lib, name, override, expected):
    assert _fwd_host_call(lib, **override) == expected, name


# attn_prefill_fp8: (q, k8, v8, k_scale, v_scale, o, lse) pointers, then the sizes; every case below
# is rejected before any CUDA call.
F8 = [0x210000, 0x220000, 0x230000, 0x240000, 0x250000, 0x260000, 0x270000]


def _prefill_fp8_call(lib, ptrs=None, B=1, Hq=4, Hkv=2, Sq=8, Skv=8, D=128, scale=0.125, causal=1):
    ptrs = F8 if ptrs is None else ptrs
    return lib.attn_prefill_fp8(*ptrs, B, Hq, Hkv, Sq, Skv, D, scale, causal, None)


PREFILL_FP8_CASES = [
    ("null k_scale", dict(ptrs=[F8[0], F8[1], F8[2], 0, F8[4], F8[5], F8[6]]), -1),
    ("null lse", dict(ptrs=F8[:6] + [0]), -1),
    ("zero query rows", dict(Sq=0), -2),
    ("causal flag 2", dict(causal=2), -2),
    ("group not integral", dict(Hq=3), -3),
    ("head dim 64", dict(D=64), -4),
    ("misaligned v8", dict(ptrs=[F8[0], F8[1], F8[2] + 4, F8[3], F8[4], F8[5], F8[6]]), -5),
    ("causal with Sq > Skv", dict(Sq=9), -6),
    ("negative scale", dict(scale=-1.0), -11),
]


@pytest.mark.parametrize("name,override,expected", PREFILL_FP8_CASES, ids=[c[0] for c in PREFILL_FP8_CASES])
def test_prefill_fp8_argument_errors(lib, name, override, expected):
    assert _prefill_fp8_call(lib, **override) == expected, name
