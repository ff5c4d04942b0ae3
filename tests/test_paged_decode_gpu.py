"""GPU parity of attn_decode_paged (single-token decode over a paged, variable-length KV cache)
against the fp64 oracle, one sequence at a time over the keys that sequence has filled.

Each case builds a dense cache per sequence from the seeded inputs, scatters its filled rows into
randomly permuted pages, fills every other row of every page with NaN (a cache's unused slots hold
anything; the decode must not let them through its PV product), and checks O and LSE of every
sequence against the oracle run on that sequence's first len_b keys. A sequence with no keys must
give O = 0 and LSE = -inf.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_attn_b200 import attn, build, inputs
from tests.compare import compare

pytestmark = pytest.mark.gpu

BF16_NAN = torch.tensor(float("nan"), dtype=torch.bfloat16)


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
    assert attn.device_status() == 0, "a kernel-side wait ran out during the paged decode tests"


def make_paged(w, lens, page_size, seed):
    """Dense seeded inputs for workload w (Skv = capacity), scattered into pages."""
    q, k, v = inputs.generate(w)
    B, Hkv, cap, D = k.shape
    pages_per_seq = -(-cap // page_size)
    num_pages = B * pages_per_seq + 3  # a few pages nobody uses
    rng = np.random.RandomState(seed)
    perm = rng.permutation(num_pages)
    table = np.full((B, pages_per_seq), num_pages + 7, dtype=np.int32)  # entries past a sequence: never read
    kp = torch.full((num_pages, Hkv, page_size, D), float("nan"), dtype=torch.bfloat16)
    vp = kp.clone()
    nxt = 0
    for b in range(B):
        for n in range(-(-lens[b] // page_size)):
            pg = int(perm[nxt])
            nxt += 1
            table[b, n] = pg
            lo, hi = n * page_size, min((n + 1) * page_size, lens[b])
            kp[pg, :, : hi - lo] = k[b, :, lo:hi]
            vp[pg, :, : hi - lo] = v[b, :, lo:hi]
    return q, k, v, kp, vp, torch.from_numpy(table), torch.tensor(lens, dtype=torch.int32)


CASES = [
    # B, Hq, Hkv, capacity, page_size, lengths, decode_ctas
    (4, 32, 8, 1000, 64, [1000, 1, 129, 0], 0),          # GQA 4, one empty sequence
    (3, 8, 8, 700, 16, [700, 127, 128], 0),              # one head per kv head, 16-key pages
    (2, 32, 2, 300, 128, [300, 256], 5),                 # 16 heads per kv head, page = chunk
    (5, 16, 4, 513, 256, [513, 1, 2, 255, 400], 1),      # a single CTA walks everything
    (6, 8, 2, 64, 32, [64, 64, 1, 0, 33, 63], 300),      # more CTAs than chunks: empty ranges
    (16, 32, 8, 4096, 128, None, 0),                     # the bench decode shape, random lengths
    (2, 4, 1, 4096, 4096, [4096, 4096], 0),              # one page per sequence: a dense cache
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_hq{}_hkv{}_cap{}_page{}_ctas{}".format(*c[:5], c[6]))
def test_paged_decode_matches_oracle(case):
    B, Hq, Hkv, cap, page_size, lens, ctas = case
    if lens is None:
        lens = [int(x) for x in np.random.RandomState(5).randint(1, cap + 1, size=B)]
    w = inputs.custom(B, Hq, Hkv, 1, cap, 128, True, seed=sum(lens) + page_size)
    q, k, v, kp, vp, table, seq_lens = make_paged(w, lens, page_size, seed=B + cap)
    o, lse = attn.attn_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), seq_lens.cuda(), max(lens),
                                    scale=w.scale, decode_ctas=ctas)
    torch.cuda.synchronize()
    o, lse = o.cpu(), lse.cpu()
    for b in range(B):
        if lens[b] == 0:
            assert torch.all(o[b] == 0), b
            assert torch.all(torch.isneginf(lse[b])), b
            continue
        o_ref, l_ref = oracle.attention(q[b:b + 1], k[b:b + 1, :, :lens[b]], v[b:b + 1, :, :lens[b]], w.scale, True)
        rep = compare(o[b:b + 1], lse[b:b + 1], o_ref, l_ref)
        assert rep.ok(), f"sequence {b} (len {lens[b]}): {rep}"


def test_paged_lengths_beyond_the_table_are_clamped():
    # seq_lens larger than the block table can hold: the decode attends to the capacity only.
    B, Hq, Hkv, cap, page_size = 2, 8, 2, 256, 64
    lens = [256, 100]
    w = inputs.custom(B, Hq, Hkv, 1, cap, 128, True, seed=77)
    q, k, v, kp, vp, table, seq_lens = make_paged(w, lens, page_size, seed=3)
    o, lse = attn.attn_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(),
                                    torch.tensor([10**6, 100], dtype=torch.int32).cuda(), 10**6, scale=w.scale)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q[:1], k[:1], v[:1], w.scale, True)
    rep = compare(o.cpu()[:1], lse.cpu()[:1], o_ref, l_ref)
    assert rep.ok(), str(rep)


def test_table_entries_outside_the_pages_read_as_zeros():
    """A block-table entry outside [0, num_pages) reads as zeros, even one whose page * Hkv would
    wrap in 32 bits onto a valid page of another sequence (2^29 + 3 with Hkv = 8 -> page 3)."""
    B, Hq, Hkv, cap, page_size = 2, 32, 8, 512, 64
    lens = [512, 300]
    w = inputs.custom(B, Hq, Hkv, 1, cap, 128, True, seed=78)
    q, k, v, kp, vp, table, seq_lens = make_paged(w, lens, page_size, seed=4)
    table[0, 2] = (1 << 29) + 3   # wraps onto page 3 if not range-checked
    table[1, 1] = -5
    o, lse = attn.attn_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), seq_lens.cuda(), max(lens),
                                    scale=w.scale)
    torch.cuda.synchronize()
    o, lse = o.cpu(), lse.cpu()
    for b, n in ((0, 2), (1, 1)):
        kz, vz = k[b:b + 1, :, :lens[b]].clone(), v[b:b + 1, :, :lens[b]].clone()
        kz[:, :, n * page_size:(n + 1) * page_size] = 0
        vz[:, :, n * page_size:(n + 1) * page_size] = 0
        o_ref, l_ref = oracle.attention(q[b:b + 1], kz, vz, w.scale, True)
        rep = compare(o[b:b + 1], lse[b:b + 1], o_ref, l_ref)
        assert rep.ok(), f"sequence {b}: {rep}"
