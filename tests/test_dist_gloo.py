"""Multi-rank host logic on CPU with the gloo backend (world sizes 2 to 4):
head sharding, max-over-ranks timing and the all-gather of per-rank results,
including uneven shards and a rank that holds no head."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from tiled_exact_attention_fa_b200 import dist as fdist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, total_bh=7):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        fdist.init("gloo", timeout_s=60)
        # each rank "took" a different time; the job time is the max
        t = fdist.max_over_ranks(1.5 + rank)
        N, d = 5, 3
        a, b = fdist.shard_range(total_bh, rank, world)
        o_full = torch.arange(total_bh * N * d, dtype=torch.float32).view(total_bh, N, d)
        l_full = torch.arange(total_bh * N, dtype=torch.float32).view(total_bh, N)
        o, l = fdist.gather_heads(o_full[a:b].clone(), l_full[a:b].clone(), total_bh)
        fdist.barrier()
        q.put((rank, t, bool(torch.equal(o, o_full)), bool(torch.equal(l, l_full)), (a, b)))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, repr(e), False, False, None))
    finally:
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world,total_bh", [(2, 7), (3, 7), (4, 3)])
def test_ranks_gloo(world, total_bh):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, total_bh)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    slowest = 1.5 + (world - 1)
    assert [r[1] for r in results] == [slowest] * world, results
    assert all(r[2] and r[3] for r in results), results
    assert [r[4] for r in results] == [fdist.shard_range(total_bh, r, world) for r in range(world)]


@pytest.mark.parametrize("total,world", [(7, 2), (64, 8), (3, 4), (2048, 3)])
def test_shard_range_partitions(total, world):
    spans = [fdist.shard_range(total, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == total
    assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_single_process_defaults():
    assert fdist.max_over_ranks(3.0) == 3.0
    fdist.barrier()
