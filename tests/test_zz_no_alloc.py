"""fa_fwd_noalloc, the entry point for callers that cannot allocate device memory.

Such callers (a serving process that has reserved all GPU memory for its own
pool, code running inside an allocator's hooks, strict per-library memory
budgets) cannot let the library cudaMalloc its workspace, so this entry point
keeps the kernel's scratch in a fixed device array instead.  Here it is
called through the C ABI twice in a row on the same stream and each result is
compared with fa_fwd's on the same inputs, with the tolerances of the other
parity tests (the two paths run the same kernel, so they normally agree bit
for bit).  The file sorts last so that a run stopping at its first failure has
already run every other test; it also passes alone in a fresh process.
"""
import math

import pytest
import torch

import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tiled_exact_attention_fa_b200 import workloads as W

pytestmark = pytest.mark.gpu

BF16_MAX_ABS = 1e-2
BF16_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def _call(entry, q, k, v, o, lse, scale, causal):
    B, H, N, d = q.shape
    stream = torch.cuda.current_stream().cuda_stream
    return int(entry(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                     B, H, N, d, scale, int(causal), fa.FA_DTYPE_BF16, stream))


@pytest.mark.parametrize("causal", [True, False])
def test_noalloc_matches_fa_fwd_twice(causal):
    fa_build.build()
    lib = fa.library()
    torch.cuda.set_device(0)
    q, k, v = (x.cuda() for x in W.random_qkv(2, 4, 1100, 128, torch.bfloat16, seed=53))
    scale = 1.0 / math.sqrt(128)

    o_ref = torch.empty_like(q)
    l_ref = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    assert _call(lib.fa_fwd, q, k, v, o_ref, l_ref, scale, causal) == fa.FA_OK, lib.fa_last_error()

    for _ in range(2):  # the shared scratch must be reusable call after call
        o = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
        rc = _call(lib.fa_fwd_noalloc, q, k, v, o, lse, scale, causal)
        assert rc == fa.FA_OK, lib.fa_last_error().decode()
        torch.cuda.synchronize()
        err = (o.float() - o_ref.float()).abs()
        assert torch.isfinite(o).all() and torch.isfinite(lse).all()
        assert err.max().item() <= BF16_MAX_ABS
        assert err.mean().item() <= BF16_MEAN_ABS
        assert (lse - l_ref).abs().max().item() <= LSE_MAX_ABS
