"""fa_fwd_host: the forward on host buffers, chunked over heads through a
copy-in / kernel / copy-out pipeline.  Its results must be bit-identical to
fa_fwd on the same inputs (the same kernels run on each head), for any
number of chunks, a ragged last chunk, pinned or pageable host memory, calls
queued back to back (staging buffers reused across calls) and staging
buffers that have to grow."""
import math

import pytest
import torch

import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tiled_exact_attention_fa_b200 import workloads as W

pytestmark = pytest.mark.gpu


def device_reference(q, k, v, scale, causal):
    o = torch.empty_like(q, device="cuda")
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    fa.forward_into(q.cuda(), k.cuda(), v.cuda(), o, lse, scale=scale, causal=causal)
    torch.cuda.synchronize()
    fa.check_device_status()
    return o.cpu(), lse.cpu()


def host_inputs(B, H, N, d, dtype, seed, pinned):
    q, k, v = W.random_qkv(B, H, N, d, dtype, seed=seed)
    if pinned:
        q, k, v = (x.pin_memory() for x in (q, k, v))
    return q, k, v


@pytest.mark.parametrize("B,H,N,d,dtype,causal", [
    (2, 9, 777, 128, torch.bfloat16, True),    # 18 heads: chunks of 3, ragged N
    (1, 3, 300, 64, torch.bfloat16, False),    # one head per chunk
    (1, 1, 1000, 128, torch.bfloat16, True),   # a single chunk
    (3, 5, 257, 64, torch.float32, True),      # fp32 kernel, 15 heads: chunks of 2, ragged last chunk
])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_path_equals_device_path(B, H, N, d, dtype, causal, pinned):
    fa_build.build()
    q, k, v = host_inputs(B, H, N, d, dtype, 83, pinned)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = device_reference(q, k, v, scale, causal)
    o = torch.full(q.shape, float("nan"), dtype=dtype, pin_memory=pinned)
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, pin_memory=pinned)
    fa.forward_host_into(q, k, v, o, lse, scale=scale, causal=causal)
    torch.cuda.current_stream().synchronize()
    fa.check_device_status()
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)


def test_back_to_back_calls_and_growing_buffers():
    fa_build.build()
    shapes = [(1, 4, 256, 128), (2, 16, 1500, 128), (1, 2, 128, 128)]  # small, larger (buffers grow), small
    cases = []
    for i, (B, H, N, d) in enumerate(shapes):
        q, k, v = host_inputs(B, H, N, d, torch.bfloat16, 90 + i, True)
        o = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True)
        cases.append((q, k, v, o, lse))
    # queue every call before synchronising once: the staging buffers are
    # reused by the next call while the previous one may still be in flight
    for rep in range(2):
        for q, k, v, o, lse in cases:
            fa.forward_host_into(q, k, v, o, lse, causal=True)
        torch.cuda.current_stream().synchronize()
        fa.check_device_status()
        for q, k, v, o, lse in cases:
            o_ref, lse_ref = device_reference(q, k, v, 1.0 / math.sqrt(q.shape[-1]), True)
            assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_forward_on_host_tensors_uses_the_host_entry():
    fa_build.build()
    q, k, v = host_inputs(1, 8, 640, 64, torch.bfloat16, 97, True)
    o, lse = fa.forward(q, k, v, causal=False)
    assert not o.is_cuda and o.is_pinned()
    o_ref, lse_ref = device_reference(q, k, v, 1.0 / 8.0, False)
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
