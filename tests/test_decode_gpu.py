"""fa_decode against the fp64 oracle: new queries over a key/value cache.

Element-by-element on every query, with the tolerances of the forward (bf16
O 1e-2 max-abs and 1e-3 mean-abs, fp32 1e-5, lse 1e-3), over cache lengths
that are not multiples of the 32-key tile, a single cached key, one to 13
queries (two query groups), causal and not, heads split into many chunks
(partials merged by the last CTA) and heads kept whole.  bf16 runs on the
warp-level MMA kernel in groups of 16 queries (cases include a full group,
a 17th query in a second group and caches shorter than one 32-key tile);
fp32 on the CUDA-core kernel."""
import math

import numpy as np
import pytest
import torch

import oracle
import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tests.parity import compare

pytestmark = pytest.mark.gpu


def make(B, H, nq, nk, d, dtype, seed, q_mult=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, H, nq, d, generator=g) * q_mult).to(dtype)
    k = torch.randn(B, H, nk, d, generator=g).to(dtype)
    v = torch.randn(B, H, nk, d, generator=g).to(dtype)
    return q, k, v


def run(q, k, v, scale, causal):
    fa_build.build()
    o = torch.full(q.shape, float("nan"), dtype=q.dtype, device="cuda")
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    fa.decode_into(q.cuda(), k.cuda(), v.cuda(), o, lse, scale=scale, causal=causal)
    torch.cuda.synchronize()
    fa.check_device_status()
    return o.cpu(), lse.cpu()


def reference(q, k, v, scale, causal):
    return oracle.attention_decode(q.float().numpy(), k.float().numpy(), v.float().numpy(), scale, causal)


CASES = [
    # B, H, nq, nk, d, causal
    (2, 4, 1, 1000, 128, False),
    (1, 2, 1, 1, 128, True),         # a single cached key
    (1, 3, 4, 777, 128, True),
    (2, 2, 8, 2050, 128, True),
    (1, 1, 13, 5000, 128, True),     # two query groups, the second ragged
    (1, 1, 1, 100_003, 128, False),  # one long head: many chunks
    (4, 8, 1, 33, 64, False),
    (1, 2, 3, 4099, 64, True),
    (3, 1, 1, 65_536, 64, True),
    # several queries run on the warp MMA in groups of 16 (bf16)
    (1, 2, 2, 300, 64, True),
    (2, 3, 16, 4000, 128, True),     # exactly one full group
    (1, 2, 17, 3000, 128, True),     # a second group of one query
    (1, 1, 16, 70_000, 64, False),   # one group, many chunks
    (2, 2, 5, 31, 128, False),       # fewer keys than one tile
]


@pytest.mark.parametrize("B,H,nq,nk,d,causal", CASES)
def test_decode_bf16_matches_oracle(B, H, nq, nk, d, causal):
    q, k, v = make(B, H, nq, nk, d, torch.bfloat16, seed=nk + 7 * nq)
    scale = 1.0 / math.sqrt(d)
    o, lse = run(q, k, v, scale, causal)
    o_ref, lse_ref = reference(q, k, v, scale, causal)
    compare(o, lse, o_ref, lse_ref, torch.bfloat16)


@pytest.mark.parametrize("B,H,nq,nk,d,causal", [(1, 2, 1, 3000, 128, False), (2, 1, 5, 700, 64, True),
                                                 (1, 1, 9, 40_000, 128, True)])
def test_decode_fp32_matches_oracle(B, H, nq, nk, d, causal):
    q, k, v = make(B, H, nq, nk, d, torch.float32, seed=3 * nk + nq)
    scale = 1.0 / math.sqrt(d)
    o, lse = run(q, k, v, scale, causal)
    o_ref, lse_ref = reference(q, k, v, scale, causal)
    compare(o, lse, o_ref, lse_ref, torch.float32)


@pytest.mark.parametrize("nq", [1, 2, 12])
def test_decode_wide_scores(nq):
    # queries scaled by 8: scores spread over ~100 natural-log units, so the
    # running max moves often and chunk partials differ by huge factors
    q, k, v = make(1, 4, nq, 20_000, 128, torch.bfloat16, seed=5, q_mult=8.0)
    o, lse = run(q, k, v, 1.0 / math.sqrt(128), True)
    o_ref, lse_ref = reference(q, k, v, 1.0 / math.sqrt(128), True)
    compare(o, lse, o_ref, lse_ref, torch.bfloat16, strict_raw=False)


def test_decode_is_the_last_rows_of_the_forward():
    # the same numbers from the two kernels: the decode of the last nq queries
    # against the whole sequence equals those rows of fa_fwd (within the
    # rounding both are allowed against the exact result)
    B, H, N, d, nq = 1, 4, 1536, 128, 5
    q, k, v = make(B, H, N, N, d, torch.bfloat16, seed=11)
    scale = 1.0 / math.sqrt(d)
    o_full = torch.empty_like(q, device="cuda")
    lse_full = torch.empty(q.shape[:3], device="cuda")
    fa.forward_into(q.cuda(), k.cuda(), v.cuda(), o_full, lse_full, scale=scale, causal=True)
    o, lse = run(q[:, :, N - nq:].contiguous(), k, v, scale, True)
    assert (o.float() - o_full[:, :, N - nq:].cpu().float()).abs().max().item() <= 2e-2
    assert (lse - lse_full[:, :, N - nq:].cpu()).abs().max().item() <= 2e-3


def test_decode_workspace_is_reused_across_sizes():
    # one cached workspace serves calls of different sizes in turn: whatever
    # a previous call left in it (other sizes' partials, counters) must not
    # matter
    shapes = [(2, 2, 3, 9000, 128), (1, 1, 1, 50_000, 64), (1, 2, 3, 4099, 64), (2, 2, 3, 9000, 128)]
    for i, (B, H, nq, nk, d) in enumerate(shapes):
        q, k, v = make(B, H, nq, nk, d, torch.bfloat16, seed=21 + i)
        assert fa.decode_workspace(B, H, nq, nk, d) is not None
        o, lse = run(q, k, v, 0.1, True)
        o2, lse2 = run(q, k, v, 0.1, True)
        assert torch.equal(o, o2) and torch.equal(lse, lse2)
        o_ref, lse_ref = reference(q, k, v, 0.1, True)
        compare(o, lse, o_ref, lse_ref, torch.bfloat16)
