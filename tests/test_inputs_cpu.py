"""The seeded-input helpers on the CPU: the paged-cache layout gathers back to the dense cache, and
the visible-pair count of a paged chunked prefill matches a brute-force count of the mask."""
import torch

from causal_attention_attn_b200 import inputs


def test_paged_cache_gathers_back_to_the_dense_rows():
    w = inputs.custom(3, 4, 2, 1, 300, 128, True, seed=3)
    _, k, v = inputs.generate(w)
    lens = [300, 17, 129]
    for page in (16, 64, 128, 256):
        kp, vp, table = inputs.paged_cache(k, v, lens, page, seed=1)
        num_pages = kp.shape[0]
        used = set()
        for b, L in enumerate(lens):
            for key in range(L):
                pg = int(table[b, key // page])
                assert 0 <= pg < num_pages
                used.add(pg)
                assert torch.equal(kp[pg, :, key % page], k[b, :, key])
                assert torch.equal(vp[pg, :, key % page], v[b, :, key])
            for n in range(-(-L // page), table.shape[1]):  # entries past the sequence point past the pages
                assert int(table[b, n]) == num_pages
        assert len(used) == sum(-(-L // page) for L in lens)  # no page shared by two sequences


def test_paged_visible_pairs_match_a_brute_force_count():
    for Sq, lens in ((256, [300, 100, 256, 0]), (5, [3, 5, 9]), (1, [1, 7])):
        brute = sum(1 for L in lens for i in range(Sq) for j in range(L) if j <= i + L - Sq)
        assert inputs.paged_visible_pairs(Sq, lens) == brute
        assert inputs.paged_visible_pairs(Sq, lens, causal=False) == Sq * sum(lens)


def test_paged_workload_lengths_are_seeded_and_in_range():
    a, b = inputs.paged_chunked_lengths(), inputs.paged_chunked_lengths()
    assert a == b and len(a) == inputs.PAGED_CHUNKED.B
    assert all(256 <= x <= 1024 for x in a)
