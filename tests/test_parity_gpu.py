"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on a B200.

Outputs are NaN-filled before each call (an unwritten row fails), and guard
bands around O and lse must come back untouched.  Every input is seeded.
"""
import math

import numpy as np
import pytest
import torch

import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tiled_exact_attention_fa_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

GUARD = 4096  # elements on each side of O and lse (keeps 16-byte alignment)
SENTINEL = 4096.0


@pytest.fixture(scope="module", autouse=True)
def _built():
    fa_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fa.library()


@pytest.fixture(autouse=True, params=[1, 2], ids=["two_tile", "one_tile"])
def forward_kernel(request, force_kernel):
    """Every test runs on each bf16 forward kernel (256-row units with two
    query tiles per CTA, and 128-row units); the f32 path ignores the choice."""
    force_kernel(request.param)
    return request.param


def run_guarded(q, k, v, scale, causal, stream=None):
    """fa_fwd through the C ABI into NaN-filled, guard-banded outputs on the GPU."""
    B, H, N, d = q.shape
    n_o, n_l = q.numel(), B * H * N
    o_buf = torch.full((n_o + 2 * GUARD,), SENTINEL, dtype=q.dtype, device=q.device)
    l_buf = torch.full((n_l + 2 * GUARD,), SENTINEL, dtype=torch.float32, device=q.device)
    o = o_buf[GUARD:GUARD + n_o].view(B, H, N, d)
    lse = l_buf[GUARD:GUARD + n_l].view(B, H, N)
    o.fill_(float("nan"))
    lse.fill_(float("nan"))
    fa.forward_into(q, k, v, o, lse, scale=scale, causal=causal, stream=stream)
    fa.check_device_status(stream)
    for buf, n in ((o_buf, n_o), (l_buf, n_l)):
        assert bool((buf[:GUARD] == SENTINEL).all()) and bool((buf[GUARD + n:] == SENTINEL).all()), \
            "write outside the output buffer"
    return o, lse


def check_against_oracle(q, k, v, scale, causal, rows=None, strict_raw=True):
    o, lse = run_guarded(q.cuda(), k.cuda(), v.cuda(), scale, causal)
    o_ref, lse_ref = parity.oracle_reference(q, k, v, scale, causal, rows)
    o, lse = o.cpu(), lse.cpu()
    if rows is not None:
        o, lse = parity.gather_rows(o, rows), parity.gather_rows(lse, rows)
    return parity.compare(o, lse, o_ref, lse_ref, q.dtype, strict_raw=strict_raw), o, lse


# ------------------------------------------------------------ small and ragged shapes

def test_first_small_bf16():
    q, k, v = W.random_qkv(1, 2, 256, 128, torch.bfloat16, seed=11)
    for causal in (False, True):
        check_against_oracle(q, k, v, 1 / math.sqrt(128), causal)


EDGE_N = [1, 2, 127, 128, 129, 200, 255, 256, 257, 383, 384, 511, 640]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", EDGE_N)
def test_bf16_edge_shapes(N, d, causal):
    q, k, v = W.random_qkv(1, 3, N, d, torch.bfloat16, seed=100 + N + d)
    check_against_oracle(q, k, v, 1 / math.sqrt(d), causal)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 31, 33, 100, 256])
def test_f32_edge_shapes(N, d, causal):
    q, k, v = W.random_qkv(2, 2, N, d, torch.float32, seed=300 + N + d)
    check_against_oracle(q, k, v, 1 / math.sqrt(d), causal)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("scale", [-0.3, 0.0, 1.0])
def test_scale_values(scale, dtype):
    q, k, v = W.random_qkv(1, 2, 300, 64, dtype, seed=17)
    # scale = 1.0 at d = 64 is 8x the usual 1/sqrt(d): rows are dominated by a
    # few keys and |O| reaches 2-4, where half a bf16 ulp of the output alone
    # is 0.0078-0.0156; as for the Q*8 workload, the max-abs bound applies to
    # the error beyond that rounding.
    strict = abs(scale) <= 0.5
    for causal in (False, True):
        check_against_oracle(q, k, v, scale, causal, strict_raw=strict)


def test_many_units_per_cta():
    # 4*40 heads x 2 query blocks = 320 work units: several per persistent CTA
    q, k, v = W.random_qkv(4, 40, 512, 128, torch.bfloat16, seed=19)
    rows = torch.arange(0, 512, 7, dtype=torch.int64).expand(4, 40, -1).contiguous()
    for causal in (False, True):
        check_against_oracle(q, k, v, 1 / math.sqrt(128), causal, rows=rows)


def test_wide_score_range_rescales():
    # Q scaled by 8 with increasing keys: the running max keeps growing
    q, k, v = W.random_qkv(1, 2, 1024, 128, torch.bfloat16, seed=23, q_mult=8.0)
    ramp = torch.linspace(0, 3, 1024).view(1, 1, 1024, 1)
    k = (k.float() + ramp).to(torch.bfloat16)
    for causal in (False, True):
        check_against_oracle(q, k, v, 1 / math.sqrt(128), causal, strict_raw=False)


# ------------------------------------------------------------ behaviour

def test_deterministic_and_stream():
    q, k, v = (x.cuda() for x in W.random_qkv(2, 4, 1000, 128, torch.bfloat16, seed=29))
    o1, l1 = run_guarded(q, k, v, 0.1, True)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o2, l2 = run_guarded(q, k, v, 0.1, True, stream=s)
    s.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 3, 640, 64, True), (2, 4, 1000, 128, False),
                                             (1, 2, 1025, 128, True), (3, 5, 129, 64, False)])
def test_both_kernels_bit_identical(B, H, N, d, causal, force_kernel):
    # same arithmetic in the same order (S, the lazily moved max, both row
    # sums, P V per block, 1/l): the two bf16 kernels agree bit for bit
    q, k, v = (x.cuda() for x in W.random_qkv(B, H, N, d, torch.bfloat16, seed=7 * N + d))
    outs = []
    for which in (1, 2):
        force_kernel(which)
        outs.append(run_guarded(q, k, v, 1 / math.sqrt(d), causal))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_causal_row0_is_exact():
    # causal row 0 sees only key 0: P = 1 exactly, so O_0 = V_0 bit for bit
    q, k, v = (x.cuda() for x in W.random_qkv(2, 3, 700, 128, torch.bfloat16, seed=31))
    o, lse = run_guarded(q, k, v, 1 / math.sqrt(128), True)
    assert torch.equal(o[:, :, 0], v[:, :, 0])
    want = (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1) / math.sqrt(128)
    assert float((lse[:, :, 0].double() - want).abs().max()) < 1e-4


def test_host_tensors_round_trip():
    q, k, v = W.random_qkv(1, 2, 384, 64, torch.bfloat16, seed=37)
    o, lse = fa.forward(q.pin_memory(), k.pin_memory(), v.pin_memory(), causal=True)
    assert not o.is_cuda and not lse.is_cuda
    o_ref, lse_ref = parity.oracle_reference(q, k, v, 1 / math.sqrt(64), True)
    parity.compare(o, lse, o_ref, lse_ref, torch.bfloat16)


def test_invalid_arguments_on_gpu():
    q = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(1, 1, 64, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.forward_into(q, q, q, q, lse)  # o aliases q
    assert e.value.status == fa.FA_ERR_INVALID_ARGUMENT
    big = torch.zeros(1, 1, 64, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.forward(big, big, big)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    fa.forward_into(q, q, q, o, lse)  # still usable after rejected calls
    fa.check_device_status()


# ------------------------------------------------------------ the five workloads

@pytest.mark.parametrize("w", W.WORKLOADS, ids=[w.name for w in W.WORKLOADS])
def test_workload(w):
    q, k, v = W.make_inputs(w)
    rows = None if w.sample_rows is None else W.sample_rows(w)
    stats, o, _ = check_against_oracle(q, k, v, w.scale, w.causal, rows=rows,
                                       strict_raw=(w.q_mult == 1.0))
    print(w.name, stats)
    if w.causal:
        # row 0 of every head (always among the checked rows, first after sorting): exact
        assert torch.equal(o[:, :, 0], v[:, :, 0])


def test_queue_reuse_over_many_launches():
    # more launches than the library has work queues: every queue is reused
    # and must have been returned to zero by the launch before
    q, k, v = (x.cuda() for x in W.random_qkv(1, 2, 300, 64, torch.bfloat16, seed=41))
    o_ref, l_ref = run_guarded(q, k, v, 0.125, True)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device="cuda")
    for _ in range(1100):
        fa.forward_into(q, k, v, o, lse, scale=0.125, causal=True)
    o.fill_(float("nan"))
    fa.forward_into(q, k, v, o, lse, scale=0.125, causal=True)
    fa.check_device_status()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_two_streams_interleaved():
    q, k, v = (x.cuda() for x in W.random_qkv(2, 8, 777, 128, torch.bfloat16, seed=43))
    ref = run_guarded(q, k, v, 0.09, False)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [(torch.empty_like(q), torch.empty(q.shape[:3], device="cuda")) for _ in range(6)]
    for i, (o, lse) in enumerate(outs):
        with torch.cuda.stream(streams[i % 2]):
            fa.forward_into(q, k, v, o, lse, scale=0.09, causal=False, stream=streams[i % 2])
    torch.cuda.synchronize()
    fa.check_device_status()
    for o, lse in outs:
        assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_growing_scores_take_the_slow_path(d, causal):
    # Scores rise by about 58 log2-units along the sequence (~7 per 128-key
    # block), so the running max of every row falls far enough behind to make
    # the kernel redo blocks against their exact max several times per row.
    N = 1024
    g = torch.Generator().manual_seed(61)
    q = torch.ones(1, 2, N, d)
    ramp = torch.linspace(0, 40.0 * 8 / d, N).view(1, 1, N, 1)
    k = (ramp + 0.05 * torch.randn(1, 2, N, d, generator=g)).expand(1, 2, N, d)
    v = torch.randn(1, 2, N, d, generator=g)
    q, k, v = (x.to(torch.bfloat16).contiguous() for x in (q, k, v))
    check_against_oracle(q, k, v, 1.0 / 8.0, causal, strict_raw=False)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("jump_at", [64, 128, 192, 320])
def test_score_jump_inside_a_block(d, jump_at):
    # Every query scores keys >= jump_at about 30 log2-units above the keys
    # before them.  A jump inside the first KV block is absorbed by the exact
    # first-block max; a jump at the start (second) half of a later block makes
    # the kernel redo that half and rescale O and l -- for the second half,
    # after the first half's P V has already been issued.
    N = 512
    g = torch.Generator().manual_seed(67)
    q = torch.ones(1, 2, N, d)
    level = torch.where(torch.arange(N) >= jump_at, 30.0 * math.log(2) * 8 / d, 0.0).view(1, 1, N, 1)
    k = level + 0.02 * torch.randn(1, 2, N, d, generator=g)
    v = torch.randn(1, 2, N, d, generator=g)
    q, k, v = (x.to(torch.bfloat16).contiguous() for x in (q, k, v))
    check_against_oracle(q, k, v, 1.0 / 8.0, False, strict_raw=False)


def test_dependent_launches_keep_stream_order():
    # The forward kernels start while the previous kernel of the stream is
    # still running and wait for it before touching memory.  A chain where
    # each forward reads the previous forward's O as its Q, with torch
    # kernels writing and reading the buffers in between, must give exactly
    # the results of the same calls with a synchronisation after each one.
    q, k, v = (x.cuda() for x in W.random_qkv(1, 4, 700, 128, torch.bfloat16, seed=97))
    scale = 1 / math.sqrt(128)

    def chain(sync):
        outs, cur = [], q
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], device="cuda")
        for i in range(12):
            o.fill_(float("nan"))                       # a torch kernel writes O first
            fa.forward_into(cur, k, v, o, lse, scale=scale, causal=i % 2 == 1)
            if sync:
                torch.cuda.synchronize()
            outs.append((o.clone(), lse.clone()))       # and one reads it right after
            cur = (o * 4.0).to(torch.bfloat16)          # the next Q comes from this O
        torch.cuda.synchronize()
        return outs

    for (o1, l1), (o2, l2) in zip(chain(False), chain(True)):
        assert not torch.isnan(o1).any()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
    fa.check_device_status()


def _random_shapes(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        out.append((int(rng.integers(1, 4)), int(rng.integers(1, 41)), int(rng.integers(1, 701)),
                    int(rng.choice([64, 128])), bool(rng.integers(0, 2))))
    return out


@pytest.mark.parametrize("B,H,N,d,causal", _random_shapes(16, 2024))
def test_random_shapes(B, H, N, d, causal):
    # seeded random shapes (B 1-3, H 1-40, N 1-700, both head dims and masks)
    # on each kernel, every row against the oracle
    q, k, v = W.random_qkv(B, H, N, d, torch.bfloat16, seed=B * 100003 + H * 1009 + N * 7 + d)
    check_against_oracle(q, k, v, 1 / math.sqrt(d), causal)


@pytest.mark.parametrize("causal", [False, True])
def test_long_sequence_sampled_rows(causal):
    # N = 2^17 + 3 rows in one head (1024 KV blocks, a ragged last one): row
    # and key offsets far past any small-size test, checked on sampled rows
    # (the first and last rows, tile edges, random rows) against the oracle
    N = (1 << 17) + 3
    q, k, v = W.random_qkv(1, 1, N, 64, torch.bfloat16, seed=131)
    g = torch.Generator().manual_seed(5)
    picks = torch.randperm(N, generator=g)[:200]
    rows = torch.cat([torch.tensor([0, 1, 127, 128, N // 2, N - 129, N - 2, N - 1]), picks]).unique().sort().values
    rows = rows.view(1, 1, -1).contiguous()
    check_against_oracle(q, k, v, 1 / 8.0, causal, rows=rows)
