"""Ring (context-parallel) attention on the CPU: the zigzag schedule (every visible block once, the
same work on every rank), and the distributed ring loop run by two and three gloo ranks against the
oracle over the whole sequence.

The ring loop (``causal_attention_attn_b200.ring.ring_attention``) is the one the GPUs run; only the
per-block compute and the merge are replaced here by CPU stand-ins: the oracle for a block's
attention (its O rounded to bf16 and its LSE to fp32, as the GPU kernel returns them) and the LSE
merge written out in fp64. The schedule, the exchange and the bookkeeping are the product's.
"""
import datetime
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_schedule_visits_each_visible_block_once():
    from causal_attention_attn_b200.ring import DIAG, FULL, ring_schedule, zigzag_chunks

    for world in range(1, 7):
        holders = {}
        for rank in range(world):
            sched = ring_schedule(rank, world)
            assert [t for t, _, _ in sched] == list(range(world))
            assert sorted(j for _, j, _ in sched) == list(range(world))  # every rank's K/V passes once
            seen = set()
            for t, j, blocks in sched:
                holders.setdefault(t, []).append(j)
                for qh, kh, mode in blocks:
                    qc, kc = zigzag_chunks(rank, world)[qh], zigzag_chunks(j, world)[kh]
                    assert mode == (DIAG if kc == qc else FULL) and kc <= qc
                    seen.add((qc, kc))
            # exactly the (query chunk, key chunk) pairs the causal mask leaves visible
            want = {(qc, kc) for qc in zigzag_chunks(rank, world) for kc in range(2 * world) if kc <= qc}
            assert seen == want
            nc = ring_schedule(rank, world, causal=False)
            assert all(mode == FULL for _, _, blocks in nc for _, _, mode in blocks)
            assert sum(len(blocks) for _, _, blocks in nc) == 4 * world
        for t, js in holders.items():  # at every step the held K/V is a permutation: one holder each
            assert sorted(js) == list(range(world))


@pytest.mark.parametrize("world", [2, 3, 4, 5, 6])
def test_zigzag_gives_every_rank_the_same_causal_work(world):
    from causal_attention_attn_b200.ring import ring_schedule, visible_pairs

    C = 64
    work = [visible_pairs(r, world, C) for r in range(world)]
    assert len(set(work)) == 1, work
    total = (2 * world * C) * (2 * world * C + 1) // 2  # the causal pairs of the whole sequence
    assert sum(work) == total
    for r in range(world):  # and the same number of blocks at every step
        assert all(len(blocks) in (2, 3) for _, _, blocks in ring_schedule(r, world))


def test_zigzag_shard_takes_chunks_r_and_2n_minus_1_minus_r():
    from causal_attention_attn_b200.ring import zigzag_shard

    x = torch.arange(12).view(1, 1, 12, 1)
    assert zigzag_shard(x, 0, 3).flatten().tolist() == [0, 1, 10, 11]
    assert zigzag_shard(x, 1, 3).flatten().tolist() == [2, 3, 8, 9]
    assert zigzag_shard(x, 2, 3).flatten().tolist() == [4, 5, 6, 7]
    with pytest.raises(ValueError):
        zigzag_shard(torch.zeros(1, 1, 10, 1), 0, 3)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _attend_cpu(q, k, v, scale, causal):
    import oracle

    o, lse = oracle.attention(q, k, v, scale, causal)
    return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(lse).to(torch.float32)


def _merge_cpu(o_acc, lse_acc, o_part, lse_part, out=None):
    # the LSE merge, in fp64: M = max, weights e^(lse - M), weighted mean of the two O's
    la, lp = lse_acc.double(), lse_part.double()
    m = torch.maximum(la, lp)
    finite = torch.isfinite(m)
    wa = torch.where(finite, torch.exp(la - torch.where(finite, m, 0.0)), torch.zeros_like(m))
    wp = torch.where(finite, torch.exp(lp - torch.where(finite, m, 0.0)), torch.zeros_like(m))
    s = wa + wp
    o = (wa[..., None] * o_acc.double() + wp[..., None] * o_part.double()) / torch.where(s > 0, s, 1.0)[..., None]
    o_acc.copy_(o.float())
    lse_acc.copy_(torch.where(s > 0, m + torch.log(torch.where(s > 0, s, 1.0)), m).float())
    if out is not None:
        out.copy_(o.to(torch.bfloat16))


def _rank_main(rank, world, port, out_dir, shape, causal):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    import oracle
    from causal_attention_attn_b200 import inputs
    from causal_attention_attn_b200.ring import ring_attention, zigzag_shard
    from tests.compare import compare

    B, Hq, Hkv, S, D = shape  # S: tokens per rank (two chunks of S / 2)
    w = inputs.custom(B, Hq, Hkv, world * S, world * S, D, causal, seed=world * 100 + S)
    q, k, v = inputs.generate(w)  # the whole sequence, the same on every rank
    o, lse = ring_attention(zigzag_shard(q, rank, world), zigzag_shard(k, rank, world),
                            zigzag_shard(v, rank, world), scale=w.scale, causal=causal, attend=_attend_cpu,
                            merge=_merge_cpu)
    ro, rl = oracle.attention(q, k, v, w.scale, causal)
    ro_r = zigzag_shard(torch.from_numpy(ro), rank, world).numpy()
    rl_r = zigzag_shard(torch.from_numpy(rl), rank, world).numpy()
    rep = compare(o, lse, ro_r, rl_r)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"ok": rep.ok(), "report": str(rep)}, f)
    dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (3, False)])
def test_ring_attention_with_gloo_matches_oracle(world, causal, tmp_path):
    import torch.multiprocessing as mp

    shape = (1, 4, 2, 24, 32)  # B, Hq, Hkv, tokens per rank (two chunks of 12), D
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), shape, causal), nprocs=world,
                       join=True, start_method="spawn")
    for r in range(world):
        with open(tmp_path / f"rank{r}.json") as f:
            res = json.load(f)
        assert res["ok"], f"rank {r}: {res['report']}"
