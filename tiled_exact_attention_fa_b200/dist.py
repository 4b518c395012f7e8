"""Multi-process plumbing for running the forward on several GPUs.

The attention forward has no exchange step: every (batch, head) and every
query row is independent (the pages tile one head's N x N problem and never
couple heads), so a multi-GPU job gives each rank its own share of the heads
(or its own batch) and runs the same kernel there.  torch.distributed is used
only to agree on timing (a barrier and a max over ranks) and, when a caller
wants the whole result on every rank, to all-gather it.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_world() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0) -> None:
    """Initialise the default process group from the environment (torchrun style)."""
    if dist.is_initialized():
        return
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))


def shard_range(total: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous share [start, stop) of `total` independent units for `rank`
    (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    """The largest `value` across ranks (the job's time is its slowest rank's)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device: torch.device | str | None = None) -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and torch.device(device).type == "cuda":
            dist.barrier(device_ids=[torch.device(device).index])
        else:
            dist.barrier()


def gather_heads(o_local: torch.Tensor, lse_local: torch.Tensor, total_bh: int):
    """All-gather per-rank [bh_r, N, d] / [bh_r, N] head shards (cut by
    shard_range) into full [total_bh, N, d] / [total_bh, N] tensors on every rank."""
    world = dist.get_world_size()
    sizes = [shard_range(total_bh, r, world) for r in range(world)]
    n_max = max(b - a for a, b in sizes)
    pad_o = o_local.new_zeros((n_max, *o_local.shape[1:]))
    pad_l = lse_local.new_zeros((n_max, *lse_local.shape[1:]))
    pad_o[: o_local.shape[0]] = o_local
    pad_l[: lse_local.shape[0]] = lse_local
    outs_o = [torch.empty_like(pad_o) for _ in range(world)]
    outs_l = [torch.empty_like(pad_l) for _ in range(world)]
    dist.all_gather(outs_o, pad_o)
    dist.all_gather(outs_l, pad_l)
    o = torch.cat([outs_o[r][: b - a] for r, (a, b) in enumerate(sizes)])
    lse = torch.cat([outs_l[r][: b - a] for r, (a, b) in enumerate(sizes)])
    return o, lse
