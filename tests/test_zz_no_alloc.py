"""fa_fwd_noalloc, the entry point for callers that cannot allocate device memory.

Such callers (a serving process that has reserved all GPU memory for its own
pool, code running inside an allocator's hooks, strict per-library memory
budgets) cannot let the library cudaMalloc its workspace, so this entry point
keeps the kernel's scratch in a fixed device array instead.  Here it is
called through the C ABI twice in a row on the same stream, for both head
dims and both dtypes, and each result is compared with the fp64 oracle (the
tolerances of the other parity tests) and with fa_fwd's result on the same
inputs.  A timeout forced by the test hook must be reported by
fa_noalloc_check_status, survive a later call, and be cleared by the check.
The file sorts last so that a run stopping at its first failure has already
run every other test; it also passes alone in a fresh process.
"""
import math

import pytest
import torch

import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tiled_exact_attention_fa_b200 import workloads as W
from tests.parity import compare, oracle_reference

pytestmark = pytest.mark.gpu

BF16_MAX_ABS = 1e-2
BF16_MEAN_ABS = 1e-3
F32_MAX_ABS = 1e-5
LSE_MAX_ABS = 1e-3


def _call(entry, q, k, v, o, lse, scale, causal):
    B, H, N, d = q.shape
    stream = torch.cuda.current_stream().cuda_stream
    dtype = fa.FA_DTYPE_BF16 if q.dtype == torch.bfloat16 else fa.FA_DTYPE_F32
    return int(entry(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                     B, H, N, d, scale, int(causal), dtype, stream))


def _outputs(q):
    o = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=q.device)
    return o, lse


@pytest.mark.parametrize("which", [0, 1, 2], ids=["by_size", "two_tile", "one_tile"])
@pytest.mark.parametrize("dtype,d,N", [(torch.bfloat16, 128, 1100), (torch.bfloat16, 64, 700),
                                       (torch.float32, 64, 300)])
@pytest.mark.parametrize("causal", [True, False])
def test_noalloc_matches_oracle_and_fa_fwd_twice(dtype, d, N, causal, which, force_kernel):
    fa_build.build()
    lib = fa.library()
    force_kernel(which)
    torch.cuda.set_device(0)
    qc, kc, vc = W.random_qkv(2, 4, N, d, dtype, seed=53 + d)
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    scale = 1.0 / math.sqrt(d)
    o_or, l_or = oracle_reference(qc, kc, vc, scale, causal)

    o_ref, l_ref = _outputs(q)
    assert _call(lib.fa_fwd, q, k, v, o_ref, l_ref, scale, causal) == fa.FA_OK, lib.fa_last_error()
    tol = BF16_MAX_ABS if dtype == torch.bfloat16 else F32_MAX_ABS

    for _ in range(2):  # the shared scratch must be reusable call after call
        o, lse = _outputs(q)
        rc = _call(lib.fa_fwd_noalloc, q, k, v, o, lse, scale, causal)
        assert rc == fa.FA_OK, lib.fa_last_error().decode()
        assert lib.fa_noalloc_check_status(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
        compare(o.cpu(), lse.cpu(), o_or, l_or, dtype)
        err = (o.float() - o_ref.float()).abs()
        assert err.max().item() <= tol
        if dtype == torch.bfloat16:
            assert err.mean().item() <= BF16_MEAN_ABS
        assert (lse - l_ref).abs().max().item() <= LSE_MAX_ABS


@pytest.mark.parametrize("which", [1, 2], ids=["two_tile", "one_tile"])
def test_noalloc_timeout_is_reported_and_cleared(which, force_kernel):
    fa_build.build()
    lib = fa.library()
    force_kernel(which)
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream().cuda_stream
    qc, kc, vc = W.random_qkv(1, 2, 512, 128, torch.bfloat16, seed=71)
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    scale = 1.0 / math.sqrt(128)
    assert lib.fa_noalloc_check_status(stream) == fa.FA_OK  # start clean
    # one CTA of the next launch skips one arrival: a bounded wait runs out (~2 s)
    assert lib.fa_test_skip_one_arrival() == fa.FA_OK
    o, lse = _outputs(q)
    assert _call(lib.fa_fwd_noalloc, q, k, v, o, lse, scale, True) == fa.FA_OK
    # a later call does not hide the timeout of the earlier one
    o2, lse2 = _outputs(q)
    assert _call(lib.fa_fwd_noalloc, q, k, v, o2, lse2, scale, True) == fa.FA_OK
    assert lib.fa_noalloc_check_status(stream) == fa.FA_ERR_DEVICE_TIMEOUT
    assert "bounded wait" in lib.fa_last_error().decode()
    # fa_fwd's own status word was not touched, and the no-alloc word is clear again
    fa.check_device_status()
    assert lib.fa_noalloc_check_status(stream) == fa.FA_OK
    # the context still works: the second call's result and a new one are right
    o_or, l_or = oracle_reference(qc, kc, vc, scale, True)
    compare(o2.cpu(), lse2.cpu(), o_or, l_or, torch.bfloat16)
    o3, lse3 = _outputs(q)
    assert _call(lib.fa_fwd_noalloc, q, k, v, o3, lse3, scale, True) == fa.FA_OK
    assert lib.fa_noalloc_check_status(stream) == fa.FA_OK
    compare(o3.cpu(), lse3.cpu(), o_or, l_or, torch.bfloat16)
