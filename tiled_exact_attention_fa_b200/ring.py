"""Sequence-parallel forward: the sequence split into one contiguous chunk
per rank, keys and values passed around a ring, partial results merged by
their log-sum-exp.

Rank r holds rows [r*n, (r+1)*n) of Q, K and V ([B, H, n, d] each).  In step
s it holds the K/V chunk c = (r - s) mod P: it attends its queries to that
chunk (fa_fwd; with the causal mask the chunk on the diagonal is the usual
causal case, chunks before it are unmasked, chunks after it are skipped) while
the chunk moves on to rank r + 1 and chunk c - 1 arrives from rank r - 1
(point-to-point sends over NCCL, posted before the kernel so they overlap
it).  After P steps the partial (o, lse) pairs are combined by fa_merge.  The
combination is exact: softmax over a union of key sets is the
log-sum-exp-weighted combination of the softmaxes over the sets -- the
online-softmax rescale ("FlashAttention, Playable", EP 04) applied to whole
chunks.  Every chunk has n keys and n queries, so fa_fwd's equal-length
contract holds for every step.

`compute` and `merge` are parameters so that the schedule can run with CPU
stand-ins on ranks that have no GPU (the gloo tests); the defaults run the
CUDA kernels.
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist


def ring_schedule(rank: int, world: int, causal: bool):
    """[(step, chunk, run, causal_block)] for one rank: which K/V chunk it
    holds at each step, whether it attends to it, and with which mask."""
    out = []
    for step in range(world):
        c = (rank - step) % world
        run = (not causal) or c <= rank
        out.append((step, c, run, causal and c == rank))
    return out


def _gpu_compute(q, k, v, causal: bool, scale):
    from tiled_exact_attention_fa_b200 import forward_into
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    forward_into(q, k, v, o, lse, scale=scale, causal=causal)
    return o, lse


def _gpu_merge(o_parts, lse_parts):
    from tiled_exact_attention_fa_b200 import merge
    return merge(o_parts, lse_parts)


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool = False,
                   scale: float | None = None, group=None,
                   compute: Callable | None = None, merge: Callable | None = None):
    """This rank's rows of the attention over the whole sequence (see the
    module docstring).  Returns (o, lse) for the local queries."""
    compute = compute or _gpu_compute
    merge = merge or _gpu_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    cur = torch.stack([k, v]).contiguous()
    parts_o, parts_l = [], []
    for step, c, run, causal_block in ring_schedule(rank, world, causal):
        reqs, nbuf = [], None
        if step < world - 1:
            nbuf = torch.empty_like(cur)
            reqs = [dist.isend(cur, nxt, group=group), dist.irecv(nbuf, prv, group=group)]
        if run:
            o_c, l_c = compute(q, cur[0], cur[1], causal_block, scale)
            parts_o.append(o_c)
            parts_l.append(l_c)
        for r in reqs:
            r.wait()
        if nbuf is not None:
            cur = nbuf
    return merge(torch.stack(parts_o), torch.stack(parts_l))


def ring_attention_emulated(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, world: int, *,
                            causal: bool = False, scale: float | None = None,
                            compute: Callable | None = None, merge: Callable | None = None):
    """The same schedule for `world` ranks run one after another in this
    process on the full sequence ([B, H, world*n, d]): for checking the
    partial-and-merge arithmetic on one GPU.  Returns the full (o, lse)."""
    compute = compute or _gpu_compute
    merge = merge or _gpu_merge
    N = q.shape[2]
    if N % world:
        raise ValueError("the sequence must split into equal chunks")
    n = N // world
    chunk = lambda t, c: t[:, :, c * n:(c + 1) * n].contiguous()
    outs_o, outs_l = [], []
    for rank in range(world):
        parts_o, parts_l = [], []
        for _, c, run, causal_block in ring_schedule(rank, world, causal):
            if run:
                o_c, l_c = compute(chunk(q, rank), chunk(k, c), chunk(v, c), causal_block, scale)
                parts_o.append(o_c)
                parts_l.append(l_c)
        o_r, l_r = merge(torch.stack(parts_o), torch.stack(parts_l))
        outs_o.append(o_r)
        outs_l.append(l_r)
    return torch.cat(outs_o, dim=2), torch.cat(outs_l, dim=2)
