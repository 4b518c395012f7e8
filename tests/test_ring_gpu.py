"""fa_merge and the sequence-parallel arithmetic on one GPU: the merge kernel
against the oracle's merge, and the zig-zag ring schedule emulated rank by
rank (fa_fwd on each chunk pair, fa_merge per query chunk) against the fp64
oracle on the whole sequence, up to the eight ranks the ring bench uses."""
import math

import numpy as np
import pytest
import torch

import oracle
import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tiled_exact_attention_fa_b200 import ring
from tests.parity import compare

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.float32, 128), (torch.bfloat16, 128)])
def test_merge_kernel_matches_oracle(dtype, d):
    fa_build.build()
    g = torch.Generator().manual_seed(3)
    P, rows = 4, 1000
    o_parts = torch.randn(P, rows, d, generator=g).to(dtype)
    lse_parts = torch.randn(P, rows, generator=g) * 5
    lse_parts[2, :100] = float("-inf")            # a part with no usable key for some rows
    lse_parts[:, 500] = float("-inf")             # a row with no usable key at all
    o, lse = fa.merge(o_parts.cuda(), lse_parts.cuda())
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.lse_merge(o_parts.float().numpy(), lse_parts.numpy())
    tol = 1e-5 if dtype == torch.float32 else 1e-2
    ok = np.isfinite(lse_ref)
    assert np.abs(o.float().cpu().numpy()[ok] - o_ref[ok]).max() <= tol
    assert np.abs(lse.cpu().numpy()[ok] - lse_ref[ok]).max() <= 1e-5
    assert torch.isinf(lse[500]).item() and lse[500].item() < 0 and (o[500] == 0).all().item()


@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_emulated_ring_matches_oracle(world, causal):
    fa_build.build()
    B, H, N, d = 1, 4, 2048, 128
    g = torch.Generator().manual_seed(world * 10 + causal)
    q, k, v = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    scale = 1.0 / math.sqrt(d)
    o, lse = ring.ring_attention_emulated(q.cuda(), k.cuda(), v.cuda(), world, causal=causal, scale=scale)
    torch.cuda.synchronize()
    fa.check_device_status()
    o_ref, lse_ref = oracle.attention_fwd(q.float().numpy(), k.float().numpy(), v.float().numpy(), scale, causal)
    compare(o.cpu(), lse.cpu(), o_ref, lse_ref, torch.bfloat16)
