"""Sequence-parallel schedule on CPU ranks (gloo, world sizes 2, 3 and 4):
the zig-zag layout, the ring of K/V pairs exchanged by one grouped
point-to-point call per step, the causal skipping and the merge, with the
fp64 oracle standing in for the CUDA kernels on each rank.  Each rank's rows
must equal the oracle's attention over the whole sequence, and every rank
must do the same work."""
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
        B, H, c, d = 1, 2, 12, 16
        q, k, v = _inputs(B, H, 2 * world * c, d, seed=9)
        ql, kl, vl = (ring.zigzag_shard(t, rank, world) for t in (q, k, v))
        o, lse = ring.ring_attention(ql, kl, vl, causal=causal, scale=0.25, compute=_cpu_compute, merge=_cpu_merge)
        import oracle
        o_ref, lse_ref = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), 0.25, causal)
        o_ref = ring.zigzag_shard(torch.from_numpy(o_ref), rank, world).numpy()
        lse_ref = ring.zigzag_shard(torch.from_numpy(lse_ref), rank, world).numpy()
        err = float(np.abs(o.numpy() - o_ref).max())
        lerr = float(np.abs(lse.numpy() - lse_ref).max())
        out.put((rank, err, lerr, None))
    except Exception as e:  # report instead of hanging the parent
        out.put((rank, None, None, repr(e)))
    finally:
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
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


def test_schedule_covers_each_chunk_pair_once():
    # Every (query chunk, key chunk) pair of the global sequence that the mask
    # leaves visible is computed exactly once, by the rank holding the query
    # chunk, with the causal mask exactly on the diagonal pairs.
    for world in (1, 2, 3, 5, 8):
        for causal in (False, True):
            seen = {}
            for rank in range(world):
                sched = ring.ring_schedule(rank, world, causal)
                assert sorted(a for _, a, _ in sched) == list(range(world))
                mine = ring.chunk_ids(rank, world)
                for _, a, calls in sched:
                    theirs = ring.chunk_ids(a, world)
                    for qp, kp, cb in calls:
                        for qi in ((0, 1) if qp == ring.ALL else (qp,)):
                            for ki in ((0, 1) if kp == ring.ALL else (kp,)):
                                gq, gk = mine[qi], theirs[ki]
                                if cb and gk > gq:
                                    continue  # fully masked inside a causal ALL call
                                assert (gq, gk) not in seen, (world, causal, gq, gk)
                                seen[(gq, gk)] = cb and gq == gk
            n = 2 * world
            want = {(x, y): causal and x == y for x in range(n) for y in range(n) if not causal or y <= x}
            assert seen == want


def test_zigzag_balances_causal_work():
    # Under the mask every rank does 2P chunk products (4P without); with
    # contiguous chunks the last rank would do 2P/(P+1) times the mean.
    for world in (1, 2, 3, 4, 8):
        for causal in (False, True):
            work = [sum(ring.call_work(c) for _, _, calls in ring.ring_schedule(r, world, causal) for c in calls)
                    for r in range(world)]
            assert work == [(2.0 if causal else 4.0) * world] * world


def test_zigzag_shard_roundtrip():
    x = torch.arange(2 * 3 * 24 * 2, dtype=torch.float32).reshape(2, 3, 24, 2)
    for world in (1, 2, 3, 4):
        parts = [ring.zigzag_shard(x, r, world) for r in range(world)]
        assert torch.equal(ring.zigzag_unshard(parts), x)
    # rank 0 of 3 holds chunks 0 and 5 (of 4 rows each)
    p0 = ring.zigzag_shard(x, 0, 3)
    assert torch.equal(p0[:, :, :4], x[:, :, :4]) and torch.equal(p0[:, :, 4:], x[:, :, 20:])
    with pytest.raises(ValueError):
        ring.zigzag_shard(x, 0, 5)


def test_emulated_ring_on_cpu():
    # the single-process emulation follows the same schedule
    q, k, v = _inputs(1, 1, 60, 8, seed=4)
    import oracle
    for world in (1, 3):
        for causal in (False, True):
            o, lse = ring.ring_attention_emulated(q, k, v, world, causal=causal, scale=0.3,
                                                  compute=_cpu_compute, merge=_cpu_merge)
            o_ref, lse_ref = oracle.attention_fwd(q.numpy(), k.numpy(), v.numpy(), 0.3, causal)
            assert np.abs(o.numpy() - o_ref).max() <= 1e-5
            assert np.abs(lse.numpy() - lse_ref).max() <= 1e-5
