"""Ring (context-parallel) attention: the sequence is cut into one contiguous chunk per rank, and
the K/V chunks travel around the ring of ranks so that every rank's queries meet every key.

Each rank r holds q, k, v of chunk r (tokens [r*S, (r+1)*S) of a sequence of world*S tokens). At
step t it holds the K/V of chunk j = (r - t) mod world and, under the causal mask, attends to it as
a full block (j < r: every key precedes every query), as the diagonal block with the causal mask
(j == r), or not at all (j > r: every key follows every query). Each block's (O, LSE) is merged
into the running result by the LSE merge, while the K/V for the next step is already in flight:
one send to rank r+1 and one receive from rank r-1 per step.

Sources (page title, section): partial results over key splits combine through their LSEs —
"AI Infra 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层优化", §3 (LSE paragraph); the
causal mask — same page, §3. The ring itself (who sends what to whom) is this library's layout.

Per block, the work runs in the library's kernels (``attn_fwd`` and ``attn_lse_merge``); the
exchange is ``torch.distributed`` point-to-point (NCCL between GPUs). ``attend`` and ``merge`` may
be replaced (the CPU tests run the same schedule with the gloo backend and a CPU stand-in).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

DIAG, FULL, SKIP = "diag", "full", "skip"


def ring_schedule(rank: int, world: int, causal: bool = True):
    """[(step, kv_chunk, mode)] for one rank: at step t it holds chunk (rank - t) mod world, and
    mode is DIAG (causal mask), FULL (no mask) or SKIP (nothing visible)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    out = []
    for t in range(world):
        j = (rank - t) % world
        if not causal:
            mode = FULL
        elif j == rank:
            mode = DIAG
        elif j < rank:
            mode = FULL
        else:
            mode = SKIP
        out.append((t, j, mode))
    return out


def _attend_gpu(q, k, v, scale, causal):
    from . import attn

    return attn.attn_fwd(q, k, v, scale=scale, causal=causal)


def _merge_gpu(o_acc, lse_acc, o_part, lse_part, out=None):
    from . import attn

    attn.attn_lse_merge(o_acc, lse_acc, o_part, lse_part, out=out)


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
                   causal: bool = True, group=None, attend=None, merge=None):
    """Attention of this rank's queries over the whole ring's keys.

    q [B, Hq, S, D], k and v [B, Hkv, S, D]: this rank's chunk (every rank the same S). Returns
    (o [B, Hq, S, D] bf16, lse [B, Hq, S] fp32), equal to rows [rank*S, (rank+1)*S) of attention
    over the concatenated sequence. Every rank of ``group`` must call it with the same shapes.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    attend = attend or _attend_gpu
    merge = merge or _merge_gpu
    if scale is None:
        scale = q.shape[-1] ** -0.5
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world

    sched = ring_schedule(rank, world, causal)
    last = max(t for t, _, mode in sched if mode != SKIP)  # the step whose merge writes the output
    o_acc = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    lse_acc = torch.full(q.shape[:-1], float("-inf"), dtype=torch.float32, device=q.device)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    kv = (k.contiguous(), v.contiguous())
    spare = (torch.empty_like(kv[0]), torch.empty_like(kv[1]))
    for t, _, mode in sched:
        reqs = []
        if t + 1 < world:  # the next step's K/V travels while this block is computed
            ops = [dist.P2POp(dist.isend, kv[0], nxt, group), dist.P2POp(dist.isend, kv[1], nxt, group),
                   dist.P2POp(dist.irecv, spare[0], prv, group), dist.P2POp(dist.irecv, spare[1], prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        if mode != SKIP:
            o_part, lse_part = attend(q, kv[0], kv[1], scale, mode == DIAG)
            merge(o_acc, lse_acc, o_part, lse_part, out if t == last else None)
        for r in reqs:
            r.wait()
        if t + 1 < world:
            kv, spare = spare, kv
    return out, lse_acc
