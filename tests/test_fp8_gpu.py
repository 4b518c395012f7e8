"""Parity of the E4M3 forward (fa_fwd_fp8, through the C ABI) with the fp64
oracle, on a B200.

The oracle computes the exact attention of the E4M3 values (upcast exactly)
with the scale scale * descale_q * descale_k, and O times descale_v (O is
linear in V).  The kernel's one approximation is P rounded to E4M3 as the
operand of P V (Q8 K8^T is exact in fp32 up to the accumulation order); each
element is held to the per-element bound derived in tests/fp8_bound.py (the
rounding of P, the bf16 output, fp32 slack), whose teeth are checked on the
CPU in tests/test_fp8_bound.py.  lse uses only fp32 arithmetic and keeps the
bf16 path's 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tiled_exact_attention_fa_b200 import workloads as W
from tests import fp8_bound, parity

pytestmark = pytest.mark.gpu

GUARD = 4096
SENTINEL = 4096.0
D = 128
LSE_MAX_ABS = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    fa_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fa.library()


def e4m3_qkv(B, H, N, seed, q_mult=1.0):
    return W.random_qkv(B, H, N, D, torch.float8_e4m3fn, seed, q_mult=q_mult)


def run_fp8(q8, k8, v8, scale, causal, dq=1.0, dk=1.0, dv=1.0):
    """fa_fwd_fp8 into NaN-filled, guard-banded bf16 / fp32 outputs."""
    B, H, N, d = q8.shape
    n_o, n_l = q8.numel(), B * H * N
    o_buf = torch.full((n_o + 2 * GUARD,), SENTINEL, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((n_l + 2 * GUARD,), SENTINEL, dtype=torch.float32, device="cuda")
    o = o_buf[GUARD:GUARD + n_o].view(B, H, N, d)
    lse = l_buf[GUARD:GUARD + n_l].view(B, H, N)
    o.fill_(float("nan"))
    lse.fill_(float("nan"))
    fa.forward_fp8_into(q8.cuda(), k8.cuda(), v8.cuda(), o, lse, descale_q=dq, descale_k=dk, descale_v=dv,
                        scale=scale, causal=causal)
    fa.check_device_status()
    for buf, n in ((o_buf, n_o), (l_buf, n_l)):
        assert bool((buf[:GUARD] == SENTINEL).all()) and bool((buf[GUARD + n:] == SENTINEL).all()), \
            "write outside the output buffer"
    return o.cpu(), lse.cpu()


def check_fp8(q8, k8, v8, scale, causal, dq=1.0, dk=1.0, dv=1.0, rows=None):
    o, lse = run_fp8(q8, k8, v8, scale, causal, dq, dk, dv)
    B, H, N, _ = q8.shape
    if rows is None:
        rows = torch.arange(N, dtype=torch.int64).expand(B, H, N).contiguous()
    o_ref, lse_ref, bound = fp8_bound.reference(q8, k8, v8, scale, causal, dq, dk, dv, rows)
    o = parity.gather_rows(o, rows).float().numpy().astype(np.float64)
    lse = parity.gather_rows(lse, rows).numpy().astype(np.float64)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), "unwritten or non-finite output"
    err = np.abs(o - o_ref)
    stats = dict(o_max_abs=float(err.max()), o_mean_abs=float(err.mean()),
                 worst_fraction_of_bound=float((err / bound).max()),
                 lse_max_abs=float(np.abs(lse - lse_ref).max()))
    assert (err <= bound).all(), stats
    assert stats["lse_max_abs"] <= LSE_MAX_ABS, stats
    return stats, o, lse


def test_first_small():
    q, k, v = e4m3_qkv(1, 2, 256, seed=11)
    for causal in (False, True):
        check_fp8(q, k, v, 1 / math.sqrt(D), causal)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 256, 257, 383, 511, 640])
def test_edge_shapes(N, causal):
    q, k, v = e4m3_qkv(1, 3, N, seed=500 + N)
    check_fp8(q, k, v, 1 / math.sqrt(D), causal)


@pytest.mark.parametrize("causal", [False, True])
def test_descale_factors(causal):
    # the three factors enter as scale * dq * dk and a multiplier of O; a
    # negative dv flips O
    q, k, v = e4m3_qkv(2, 2, 384, seed=71)
    check_fp8(q, k, v, 1 / math.sqrt(D), causal, dq=0.5, dk=3.0, dv=-0.25)


def test_negative_scale():
    q, k, v = e4m3_qkv(1, 2, 300, seed=73)
    check_fp8(q, k, v, -1 / math.sqrt(D), True)


def test_wide_scores():
    # Q * 8 spreads the scores over tens of log2 units, so later blocks often
    # exceed the running max by more than 8 log2 units: the max moves and O
    # and l are rescaled
    q, k, v = e4m3_qkv(1, 4, 1024, seed=79, q_mult=8.0)
    check_fp8(q, k, v, 1 / math.sqrt(D), True)


@pytest.mark.parametrize("jump_at", [64, 320])
def test_score_jump(jump_at):
    # every query scores keys >= jump_at ~29 log2 units above the ones before
    # them: inside the first block it sets the exact max; in a later block it
    # moves the running max and rescales O and l
    N = 512
    g = torch.Generator().manual_seed(83)
    q = torch.ones(1, 2, N, D)
    level = torch.where(torch.arange(N) >= jump_at, 1.25, 0.0).view(1, 1, N, 1)
    k = level + 0.02 * torch.randn(1, 2, N, D, generator=g)
    v = torch.randn(1, 2, N, D, generator=g)
    q, k, v = (x.to(torch.float8_e4m3fn).contiguous() for x in (q, k, v))
    check_fp8(q, k, v, 1.0 / 8.0, False)


def test_causal_row0_is_v0_exactly():
    # row 0 sees one key: p = 1 exactly, O_0 = V8_0 (E4M3 values are exact in bf16)
    q, k, v = e4m3_qkv(2, 3, 384, seed=89)
    o, lse = run_fp8(q, k, v, 1 / math.sqrt(D), True)
    assert torch.equal(o[:, :, 0], v[:, :, 0].to(torch.bfloat16))
    s00 = (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1) / math.sqrt(D)
    assert torch.allclose(lse[:, :, 0].double(), s00, rtol=0, atol=1e-5)


@pytest.mark.parametrize("w", W.FP8_WORKLOADS, ids=[w.name for w in W.FP8_WORKLOADS])
def test_workloads(w):
    q, k, v = W.make_inputs(w)
    stats, _, _ = check_fp8(q, k, v, w.scale, w.causal, rows=W.sample_rows(w))
    print(w.name, stats)


@pytest.mark.parametrize("causal", [False, True])
def test_host_buffers_match_device_path(causal):
    # fa_fwd_fp8_host (pinned host tensors, chunks of heads through the
    # copy/kernel/copy pipeline) gives the device path's result bit for bit;
    # 2 x 9 heads make several chunks, N = 700 a ragged last tile
    q, k, v = e4m3_qkv(2, 9, 700, seed=71)
    o_d, l_d = fa.forward_fp8(q.cuda(), k.cuda(), v.cuda(), descale_v=0.5, causal=causal)
    o_h, l_h = fa.forward_fp8(q.pin_memory(), k.pin_memory(), v.pin_memory(), descale_v=0.5, causal=causal)
    fa.check_device_status()
    assert not o_h.is_cuda
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(l_h, l_d.cpu())
