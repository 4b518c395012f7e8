"""Sequence-parallel forward: one sequence spread over P ranks, keys and
values passed around a ring, partial results merged by their log-sum-exp.

Layout (zig-zag).  The sequence of N rows is cut into 2P chunks of c = N/2P
rows; rank r holds chunks r and 2P-1-r, concatenated in that order, of Q, K
and V ([B, H, 2c, d] each; `zigzag_shard` cuts them, `zigzag_unshard` puts
per-rank results back in sequence order).  Under the causal mask every rank
then has the same work: one early and one late chunk of queries.  With
contiguous chunks the last rank would see every key and the first only its
own, about 2P/(P+1) times the balanced share on the slowest rank.

Steps.  In step s rank r holds the K/V pair of rank a = (r - s) mod P.  It
hands that pair on to rank r + 1 and receives the next one from rank r - 1
in ONE grouped point-to-point call (`dist.batch_isend_irecv`: both directions
are posted together, so no rank's send can block its own receive when r + 1
and r - 1 are the same rank), and meanwhile attends its queries to the pair
it holds:
  * a == r: the local 2c x 2c problem, causal (the two chunks keep their
    sequence order, so the causal mask on the concatenation is the global
    one);
  * a <  r: both query chunks see key chunk a in full and nothing of chunk
    2P-1-a (it lies after both);
  * a >  r: only the late query chunk 2P-1-r sees keys, and it sees both
    chunks of the pair in full.
Without the mask every step is one unmasked 2c x 2c call.  Each rank does 2P
chunk-by-chunk products under the mask (4P without), whatever its rank.

The partial (o, lse) of each query chunk are combined by fa_merge.  The
combination is exact: softmax over a union of key sets is the
log-sum-exp-weighted combination of the softmaxes over the sets -- the
online-softmax rescale ("FlashAttention, Playable", EP 04) applied to whole
chunks.  Every call pairs equal-length chunks, so fa_fwd's contract (as many
keys as queries) holds throughout.

`compute` and `merge` are parameters so that the schedule can run with CPU
stand-ins on ranks that have no GPU (the gloo tests); the defaults run the
CUDA kernels.
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist

ALL = "all"  # the whole local 2c rows, in their zig-zag order


def chunk_ids(rank: int, world: int) -> tuple[int, int]:
    """Global chunk indices (of 2*world) held by `rank`, in local order."""
    return rank, 2 * world - 1 - rank


def ring_schedule(rank: int, world: int, causal: bool):
    """[(step, src, calls)] for one rank: in each step the rank whose K/V
    pair it holds and the products it computes with it.  A call is
    (query part, key part, causal) where a part is ALL (the local 2c rows)
    or a local chunk index 0 / 1."""
    out = []
    for step in range(world):
        a = (rank - step) % world
        if not causal:
            calls = [(ALL, ALL, False)]
        elif a == rank:
            calls = [(ALL, ALL, True)]
        elif a < rank:
            calls = [(0, 0, False), (1, 0, False)]
        else:
            calls = [(1, 0, False), (1, 1, False)]
        out.append((step, a, calls))
    return out


def call_work(call) -> float:
    """Work of one call in units of one unmasked chunk-by-chunk product."""
    qp, kp, causal = call
    size = (2 if qp == ALL else 1) * (2 if kp == ALL else 1)
    return size / 2 if causal else float(size)


def zigzag_shard(x: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """This rank's rows of a [B, H, N, d] (or [B, H, N]) tensor: chunks r and
    2P-1-r of 2P, concatenated (contiguous copy)."""
    N = x.shape[2]
    if N % (2 * world):
        raise ValueError("the sequence must split into 2 * world equal chunks")
    c = N // (2 * world)
    lo, hi = chunk_ids(rank, world)
    return torch.cat([x[:, :, lo * c:(lo + 1) * c], x[:, :, hi * c:(hi + 1) * c]], dim=2).contiguous()


def zigzag_unshard(parts: list[torch.Tensor]) -> torch.Tensor:
    """Inverse of zigzag_shard over all ranks: per-rank [B, H, 2c, ...]
    tensors (rank order) back to the [B, H, N, ...] sequence order."""
    world = len(parts)
    c = parts[0].shape[2] // 2
    chunks = [None] * (2 * world)
    for r, t in enumerate(parts):
        lo, hi = chunk_ids(r, world)
        chunks[lo] = t[:, :, :c]
        chunks[hi] = t[:, :, c:]
    return torch.cat(chunks, dim=2)


def _gpu_compute(q, k, v, causal: bool, scale):
    from tiled_exact_attention_fa_b200 import forward_into
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    forward_into(q, k, v, o, lse, scale=scale, causal=causal)
    return o, lse


def _gpu_merge(o_parts, lse_parts):
    from tiled_exact_attention_fa_b200 import merge
    return merge(o_parts, lse_parts)


def _split(x: torch.Tensor) -> list[torch.Tensor]:
    """The two local chunks of a [B, H, 2c, ...] tensor as contiguous tensors."""
    c = x.shape[2] // 2
    return [x[:, :, :c].contiguous(), x[:, :, c:].contiguous()]


def _run_calls(q, kv_full, kv_chunks, q_chunks, calls, causal_mode, scale, compute, parts):
    """The calls of one step; partial results are appended per query chunk
    (parts[0], parts[1]) or, for ALL-rows calls, to parts[ALL]."""
    for qp, kp, cb in calls:
        if qp == ALL:
            k, v = kv_full
            parts[ALL].append(compute(q, k, v, cb, scale))
        else:
            k, v = kv_chunks[0][kp], kv_chunks[1][kp]
            parts[qp].append(compute(q_chunks[qp], k, v, cb, scale))


def _merge_parts(parts, merge):
    """(o, lse) for the local 2c rows from the per-chunk and whole-rows parts."""
    if not parts[0] and not parts[1]:
        return merge(torch.stack([o for o, _ in parts[ALL]]), torch.stack([l for _, l in parts[ALL]]))
    c = parts[ALL][0][0].shape[2] // 2
    outs_o, outs_l = [], []
    for x in (0, 1):
        os_ = [o[:, :, x * c:(x + 1) * c] for o, _ in parts[ALL]] + [o for o, _ in parts[x]]
        ls_ = [l[:, :, x * c:(x + 1) * c] for _, l in parts[ALL]] + [l for _, l in parts[x]]
        o_x, l_x = merge(torch.stack(os_), torch.stack(ls_))
        outs_o.append(o_x)
        outs_l.append(l_x)
    return torch.cat(outs_o, dim=2), torch.cat(outs_l, dim=2)


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool = False,
                   scale: float | None = None, group=None,
                   compute: Callable | None = None, merge: Callable | None = None):
    """This rank's rows of the attention over the whole sequence (see the
    module docstring for the zig-zag layout of q, k, v and of the result).
    Returns (o, lse) for the local 2c queries, in the local order."""
    compute = compute or _gpu_compute
    merge = merge or _gpu_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if q.shape[2] % 2:
        raise ValueError("each rank holds two equal chunks: the local length must be even")
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    # Under the mask the pair travels as two contiguous chunks (the calls use
    # one chunk at a time); without it as the local [B, H, 2c, d] tensors.
    cur = [torch.stack(_split(k)), torch.stack(_split(v))] if causal else [k, v]
    q_chunks = _split(q) if causal else None
    parts = {ALL: [], 0: [], 1: []}
    for step, _, calls in ring_schedule(rank, world, causal):
        reqs, nbuf = [], None
        if step < world - 1:
            nbuf = [torch.empty_like(t) for t in cur]
            ops = [dist.P2POp(dist.isend, cur[0], nxt, group), dist.P2POp(dist.isend, cur[1], nxt, group),
                   dist.P2POp(dist.irecv, nbuf[0], prv, group), dist.P2POp(dist.irecv, nbuf[1], prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        if step == 0:
            kv_full = (k, v)
        else:
            kv_full = (cur[0], cur[1]) if not causal else None
        _run_calls(q, kv_full, cur, q_chunks, calls, causal, scale, compute, parts)
        for r in reqs:
            r.wait()
        if nbuf is not None:
            cur = nbuf
    return _merge_parts(parts, merge)


def ring_attention_emulated(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, world: int, *,
                            causal: bool = False, scale: float | None = None,
                            compute: Callable | None = None, merge: Callable | None = None):
    """The same schedule for `world` ranks run one after another in this
    process on the full sequence ([B, H, N, d], N a multiple of 2 * world):
    for checking the partial-and-merge arithmetic on one GPU.  Returns the
    full (o, lse) in sequence order."""
    compute = compute or _gpu_compute
    merge = merge or _gpu_merge
    local = [[zigzag_shard(t, r, world) for t in (q, k, v)] for r in range(world)]
    outs_o, outs_l = [], []
    for rank in range(world):
        ql = local[rank][0]
        q_chunks = _split(ql) if causal else None
        parts = {ALL: [], 0: [], 1: []}
        for _, a, calls in ring_schedule(rank, world, causal):
            ka, va = local[a][1], local[a][2]
            kv_chunks = [torch.stack(_split(ka)), torch.stack(_split(va))] if causal else None
            _run_calls(ql, (ka, va), kv_chunks, q_chunks, calls, causal, scale, compute, parts)
        o_r, l_r = _merge_parts(parts, merge)
        outs_o.append(o_r)
        outs_l.append(l_r)
    return zigzag_unshard(outs_o), zigzag_unshard(outs_l)
