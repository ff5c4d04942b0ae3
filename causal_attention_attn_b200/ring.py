"""Ring (context-parallel) attention: each rank holds part of one long sequence, and the K/V parts
travel around the ring of ranks so that every rank's queries meet every key.

Layout (zigzag): a sequence of 2*world*C tokens is cut into 2*world chunks of C tokens, and rank r
holds chunk r and chunk 2*world-1-r, in that order ([lo | hi], 2*C tokens; ``zigzag_shard``). Under
the causal mask a contiguous split would give rank r r+1 blocks of work; pairing an early chunk
with a late one gives every rank the same work: 2*C*C visible pairs per step, plus C on its own
step. At step t rank r holds the K/V of rank j = (r - t) mod world and attends to it block by
block, a block being (query chunk, key chunk): full when the key chunk precedes the query chunk,
the diagonal block with the causal mask when they are the same chunk, skipped when it follows:

    j == r:  (lo, lo) diagonal, (hi, lo) full, (hi, hi) diagonal
    j <  r:  (lo, lo) full,     (hi, lo) full          (j's hi chunk follows both query chunks)
    j >  r:  (hi, lo) full,     (hi, hi) full          (both of j's chunks follow r's lo chunk)

Each block's (O, LSE) is merged by the LSE merge into the running result of its query chunk, while
the K/V for the next step is already in flight: one send to rank r+1 and one receive from rank r-1
per step.

Sources (page title, section): partial results over key splits combine through their LSEs —
"AI Infra 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层优化", §3 (LSE paragraph); the
causal mask — same page, §3. The ring and the zigzag chunk order are this library's layout.

Per block, the work runs in the library's kernels (``attn_fwd`` and ``attn_lse_merge``); the
exchange is ``torch.distributed`` point-to-point (NCCL between GPUs). Splitting the rank's tokens
into its two chunks and joining the two results are plain copies. ``attend`` and ``merge`` may be
replaced (the CPU tests run the same schedule with the gloo backend and a CPU stand-in).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

DIAG, FULL = "diag", "full"
LO, HI = 0, 1  # the two chunks a rank holds


def zigzag_chunks(rank: int, world: int):
    """The chunk indices (lo, hi) rank `rank` holds: `rank` and `2*world - 1 - rank`."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank, 2 * world - 1 - rank


def zigzag_shard(x: torch.Tensor, rank: int, world: int, dim: int = 2) -> torch.Tensor:
    """Rank `rank`'s part of a whole-sequence tensor: its two chunks along `dim`, concatenated."""
    n = x.shape[dim]
    if n % (2 * world):
        raise ValueError(f"sequence length {n} is not a multiple of 2 * world = {2 * world}")
    c = n // (2 * world)
    lo, hi = zigzag_chunks(rank, world)
    return torch.cat([x.narrow(dim, lo * c, c), x.narrow(dim, hi * c, c)], dim=dim).contiguous()


def ring_schedule(rank: int, world: int, causal: bool = True):
    """[(step, source_rank, blocks)] for one rank. At step t it holds the K/V chunks of rank
    source_rank = (rank - t) mod world; blocks lists (query_half, key_half, mode) with halves LO/HI
    and mode DIAG (causal mask) or FULL (no mask); blocks with no visible key are left out."""
    out = []
    for t in range(world):
        j = (rank - t) % world
        blocks = []
        for qh, qc in enumerate(zigzag_chunks(rank, world)):
            for kh, kc in enumerate(zigzag_chunks(j, world)):
                if not causal or kc < qc:
                    blocks.append((qh, kh, FULL))
                elif kc == qc:
                    blocks.append((qh, kh, DIAG))
        out.append((t, j, blocks))
    return out


def visible_pairs(rank: int, world: int, chunk: int, causal: bool = True) -> int:
    """(query, key) pairs rank `rank` attends to over the whole ring, with chunks of `chunk` tokens."""
    diag = chunk * (chunk + 1) // 2
    return sum(diag if mode == DIAG else chunk * chunk
               for _, _, blocks in ring_schedule(rank, world, causal) for _, _, mode in blocks)


def _attend_gpu(q, k, v, scale, causal):
    from . import attn

    return attn.attn_fwd(q, k, v, scale=scale, causal=causal)


def _merge_gpu(o_acc, lse_acc, o_part, lse_part, out=None):
    from . import attn

    attn.attn_lse_merge(o_acc, lse_acc, o_part, lse_part, out=out)


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
                   causal: bool = True, group=None, attend=None, merge=None):
    """Attention of this rank's queries over the whole ring's keys.

    q [B, Hq, 2C, D], k and v [B, Hkv, 2C, D]: this rank's two chunks in zigzag order (see
    ``zigzag_shard``; every rank the same C). Returns (o [B, Hq, 2C, D] bf16, lse [B, Hq, 2C] fp32)
    in the same order: the rows of this rank's chunks of attention over the whole sequence. Every
    rank of ``group`` must call it with the same shapes.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    attend = attend or _attend_gpu
    merge = merge or _merge_gpu
    if scale is None:
        scale = q.shape[-1] ** -0.5
    n = q.shape[2]
    if n % 2 or k.shape[2] != n or v.shape[2] != n:
        raise ValueError("q, k and v must hold the same even number of tokens (two chunks)")
    c = n // 2
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world

    def halves(x):
        return x[:, :, :c].contiguous(), x[:, :, c:].contiguous()

    qs = halves(q)
    kv = [*halves(k), *halves(v)]  # k_lo, k_hi, v_lo, v_hi: what travels
    spare = [torch.empty_like(t) for t in kv]
    sched = ring_schedule(rank, world, causal)
    last = {}  # the (step, block) whose merge writes each query half's output
    for t, _, blocks in sched:
        for b, (qh, _, _) in enumerate(blocks):
            last[qh] = (t, b)
    o_acc = [torch.zeros(x.shape, dtype=torch.float32, device=q.device) for x in qs]
    lse_acc = [torch.full(x.shape[:-1], float("-inf"), dtype=torch.float32, device=q.device) for x in qs]
    out = [torch.empty(x.shape, dtype=torch.bfloat16, device=q.device) for x in qs]
    for t, _, blocks in sched:
        reqs = []
        if t + 1 < world:  # the next step's K/V travels while this step's blocks are computed
            ops = [dist.P2POp(dist.isend, x, nxt, group) for x in kv] + \
                  [dist.P2POp(dist.irecv, x, prv, group) for x in spare]
            reqs = dist.batch_isend_irecv(ops)
        for b, (qh, kh, mode) in enumerate(blocks):
            o_part, lse_part = attend(qs[qh], kv[kh], kv[2 + kh], scale, mode == DIAG)
            merge(o_acc[qh], lse_acc[qh], o_part, lse_part, out[qh] if last[qh] == (t, b) else None)
        for r in reqs:
            r.wait()
        if t + 1 < world:
            kv, spare = spare, kv
    return torch.cat(out, dim=2), torch.cat(lse_acc, dim=2)
