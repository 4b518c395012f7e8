"""Sequence-parallel schedule on CPU ranks (gloo, world sizes 2 and 3): the
ring of K/V chunks, the causal skipping and the merge, with the fp64 oracle
standing in for the CUDA kernels on each rank.  Each rank's rows must equal
the oracle's attention over the whole sequence."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tiled_exact_attention_fa_b200 import ring


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return tuple(torch.randn(B, H, N, d, generator=g) for _ in range(3))


def _cpu_compute(q, k, v, causal, scale):
    import oracle
    o, lse = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), scale, causal)
    return torch.from_numpy(o.astype(np.float32)), torch.from_numpy(lse.astype(np.float32))


def _cpu_merge(o_parts, lse_parts):
    import oracle
    o, lse = oracle.lse_merge(o_parts.numpy(), lse_parts.numpy())
    return torch.from_numpy(o.astype(np.float32)), torch.from_numpy(lse.astype(np.float32))


def _worker(rank, world, port, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    try:
        torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
        B, H, n, d = 1, 2, 24, 16
        q, k, v = _inputs(B, H, world * n, d, seed=9)
        sl = slice(rank * n, (rank + 1) * n)
        o, lse = ring.ring_attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(),
                                     causal=causal, scale=0.25, compute=_cpu_compute, merge=_cpu_merge)
        import oracle
        o_ref, lse_ref = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), 0.25, causal)
        err = float(np.abs(o.numpy() - o_ref[:, :, sl]).max())
        lerr = float(np.abs(lse.numpy() - lse_ref[:, :, sl]).max())
        out.put((rank, err, lerr, None))
    except Exception as e:  # report instead of hanging the parent
        out.put((rank, None, None, repr(e)))
    finally:
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_matches_whole_sequence(world, causal):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    for rank, err, lerr, exc in results:
        assert exc is None, exc
        assert err <= 1e-5 and lerr <= 1e-5, (rank, err, lerr)


def test_schedule_covers_each_chunk_once():
    for world in (1, 2, 5):
        for causal in (False, True):
            for rank in range(world):
                sched = ring.ring_schedule(rank, world, causal)
                assert sorted(c for _, c, _, _ in sched) == list(range(world))
                used = [c for _, c, run, _ in sched if run]
                assert sorted(used) == (list(range(rank + 1)) if causal else list(range(world)))
                assert [c for _, c, _, cb in sched if cb] == ([rank] if causal else [])


def test_emulated_ring_on_cpu():
    # the single-process emulation follows the same schedule
    q, k, v = _inputs(1, 1, 60, 8, seed=4)
    import oracle
    for causal in (False, True):
        o, lse = ring.ring_attention_emulated(q, k, v, 3, causal=causal, scale=0.3,
                                              compute=_cpu_compute, merge=_cpu_merge)
        o_ref, lse_ref = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), 0.3, causal)
        assert np.abs(o.numpy() - o_ref).max() <= 1e-5
        assert np.abs(lse.numpy() - lse_ref).max() <= 1e-5
