"""GPU parity of attn_prefill_paged (chunked prefill over a paged, variable-length KV cache) against
the fp64 oracle, one sequence at a time over the keys that sequence has filled.

Each case builds a dense cache per sequence from the seeded inputs, scatters each sequence's first
len_b rows into randomly permuted pages and fills every other slot of every page with NaN (unused
cache slots hold anything). Sequence b's Sq query rows are the last Sq tokens of its len_b keys, so
under the causal mask query i sees key j iff j <= i + len_b - Sq; the oracle gets exactly that
(its own bottom-right alignment over the sequence's len_b keys). A row that sees no key must give
O = 0 and LSE = -inf. Tolerance (tests/compare.py): O max|err| <= 1e-2, mean <= 1e-3, LSE <= 1e-3.
"""
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
    if torch.cuda.get_device_capability(0) != (10, 0):
        pytest.skip("needs an sm_100 device")
    build.build()
    attn.load_library()
    yield
    torch.cuda.synchronize()
    assert attn.device_status() == 0, "a kernel-side wait ran out during the paged prefill tests"


def make_pages(k, v, lens, page_size, seed):
    B, Hkv, cap, D = k.shape
    pages_per_seq = -(-cap // page_size)
    num_pages = B * pages_per_seq + 3
    perm = np.random.RandomState(seed).permutation(num_pages)
    table = np.full((B, pages_per_seq), num_pages + 7, dtype=np.int32)  # entries past a sequence: never read
    kp = torch.full((num_pages, Hkv, page_size, D), float("nan"), dtype=torch.bfloat16)
    vp = kp.clone()
    nxt = 0
    for b in range(B):
        for n in range(-(-min(lens[b], cap) // page_size)):
            pg = int(perm[nxt])
            nxt += 1
            table[b, n] = pg
            lo, hi = n * page_size, min((n + 1) * page_size, lens[b])
            kp[pg, :, :hi - lo] = k[b, :, lo:hi]
            vp[pg, :, :hi - lo] = v[b, :, lo:hi]
    return kp, vp, torch.from_numpy(table)


def expected(q, k, v, b, L, scale, causal):
    """Oracle O and LSE of sequence b over its first L keys; rows that see no key: 0 and -inf."""
    _, Hq, Sq, D = q.shape
    o = np.zeros((1, Hq, Sq, D))
    lse = np.full((1, Hq, Sq), -np.inf)
    if L == 0:
        return o, lse
    first = max(0, Sq - L) if causal else 0  # rows before it see no key under the mask
    ro, rl = oracle.attention(q[b:b + 1, :, first:].contiguous(), k[b:b + 1, :, :L].contiguous(),
                              v[b:b + 1, :, :L].contiguous(), scale, causal)
    o[:, :, first:] = ro
    lse[:, :, first:] = rl
    return o, lse


def check_case(B, Hq, Hkv, Sq, cap, page_size, lens, causal, seed, table_edit=None, max_seq_len=None):
    w = inputs.custom(B, Hq, Hkv, Sq, cap, 128, causal, seed=seed)
    q, k, v = inputs.generate(w)  # q [B, Hq, Sq, D]; k, v [B, Hkv, cap, D]
    kp, vp, table = make_pages(k, v, lens, page_size, seed=seed + 1)
    if table_edit is not None:
        table_edit(table, k, v)
    seq = torch.tensor(lens, dtype=torch.int32)
    o, lse = attn.attn_prefill_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), seq.cuda(),
                                     max_seq_len if max_seq_len is not None else max(lens), scale=w.scale,
                                     causal=causal)
    torch.cuda.synchronize()
    o, lse = o.cpu(), lse.cpu()
    for b in range(B):
        L = min(lens[b], cap, max_seq_len if max_seq_len is not None else max(lens))
        eo, el = expected(q, k, v, b, L, w.scale, causal)
        empty = np.isneginf(el)
        got_l = lse[b:b + 1].numpy().astype(np.float64)
        assert np.array_equal(np.isneginf(got_l), empty), f"sequence {b}: rows without keys differ"
        assert torch.all(o[b:b + 1][torch.from_numpy(empty)] == 0), f"sequence {b}: rows without keys not zero"
        if (~empty).any():
            rep = compare(o[b:b + 1][torch.from_numpy(~empty)], lse[b:b + 1][torch.from_numpy(~empty)],
                          eo[~empty], el[~empty])
            assert rep.ok(), f"sequence {b} (len {L}): {rep}"


CASES = [
    # B, Hq, Hkv, Sq, capacity, page_size, lengths, causal
    (8, 32, 8, 256, 1024, 128, [768, 300, 512, 1024, 256, 640, 385, 999], True),   # chunked prefill, ragged
    (3, 8, 2, 100, 400, 16, [400, 100, 157], True),                                 # 16-key pages
    (4, 6, 2, 130, 512, 64, [512, 129, 0, 200], True),                              # odd group, len < Sq, empty
    (2, 4, 4, 64, 700, 256, [700, 65], False),                                      # non-causal, 256-key pages
    (2, 16, 2, 300, 2048, 32, [2048, 1000], True),                                  # long, 32-key pages
    # 72 (batch, query-tile) pairs: more than the kernel puts in order of their real KV-tile counts,
    # so the work list keeps the equal-length order
    (9, 4, 2, 1024, 1100, 64, [1100, 1024, 1050, 1080, 1024, 1099, 1070, 1030, 1060], True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_hq{}_hkv{}_sq{}_cap{}_page{}_{}".format(
    *c[:6], "c" if c[7] else "nc"))
def test_paged_prefill_matches_oracle(case):
    B, Hq, Hkv, Sq, cap, page_size, lens, causal = case
    check_case(B, Hq, Hkv, Sq, cap, page_size, lens, causal, seed=sum(lens) + page_size)


def test_paged_prefill_with_one_page_per_sequence_equals_attn_fwd_bitwise():
    """Pages as large as the sequences hold a dense cache: same bits as attn_fwd."""
    w = inputs.custom(2, 8, 2, 256, 768, 128, True, seed=41)
    q, k, v = inputs.generate(w)
    kp, vp, table = make_pages(k, v, [768, 768], 768, seed=3)
    o, lse = attn.attn_prefill_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(),
                                     torch.tensor([768, 768], dtype=torch.int32).cuda(), 768, scale=w.scale)
    o_ref, l_ref = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=w.scale, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_lengths_beyond_the_table_are_clamped_and_bad_entries_read_as_zeros():
    """seq_lens larger than the table holds attend to the capacity only; an entry outside
    [0, num_pages), even one that would wrap page * Hkv in 32 bits, reads as zeros."""
    B, Hq, Hkv, Sq, cap, page = 2, 8, 8, 128, 512, 128

    def edit(table, k, v):
        table[1, 1] = (1 << 29) + 3
        k[1, :, 128:256] = 0
        v[1, :, 128:256] = 0

    w = inputs.custom(B, Hq, Hkv, Sq, cap, 128, True, seed=77)
    q, k, v = inputs.generate(w)
    kp, vp, table = make_pages(k, v, [512, 400], page, seed=9)
    edit(table, k, v)
    o, lse = attn.attn_prefill_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(),
                                     torch.tensor([10**6, 400], dtype=torch.int32).cuda(), 10**6, scale=w.scale)
    torch.cuda.synchronize()
    for b, L in ((0, 512), (1, 400)):
        eo, el = expected(q, k, v, b, L, w.scale, True)
        rep = compare(o.cpu()[b:b + 1], lse.cpu()[b:b + 1], eo, el)
        assert rep.ok(), f"sequence {b}: {rep}"


def test_paged_prefill_writes_only_in_bounds():
    """o and lse inside sentinel-filled buffers: every sentinel survives."""
    B, Hq, Hkv, Sq, cap, page = 2, 4, 2, 200, 333, 64
    w = inputs.custom(B, Hq, Hkv, Sq, cap, 128, True, seed=12)
    q, k, v = inputs.generate(w)
    kp, vp, table = make_pages(k, v, [333, 150], page, seed=5)
    pad = 4096
    n = q.numel()
    obuf = torch.full((2 * pad + n,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((2 * pad + B * Hq * Sq,), 7.0, dtype=torch.float32, device="cuda")
    o = obuf[pad:pad + n].view(q.shape)
    lse = lbuf[pad:pad + B * Hq * Sq].view(B, Hq, Sq)
    attn.attn_prefill_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), torch.tensor([333, 150], dtype=torch.int32).cuda(),
                            333, scale=w.scale, out=o, lse=lse)
    torch.cuda.synchronize()
    assert (obuf[:pad] == 7.0).all() and (obuf[pad + n:] == 7.0).all()
    assert (lbuf[:pad] == 7.0).all() and (lbuf[pad + B * Hq * Sq:] == 7.0).all()
