"""Parity of the E4M3 forward (fa_fwd_fp8, through the C ABI) with the fp64
oracle, on a B200.

The oracle computes the exact attention of the E4M3 values (upcast exactly)
with the scale scale * descale_q * descale_k, and O times descale_v (O is
linear in V).  The kernel's one approximation is P rounded to E4M3 as the
operand of P V (Q8 K8^T is exact in fp32 up to the accumulation order).  E4M3
round-to-nearest has a relative error of at most 2^-4 for normal values (3
mantissa bits) and an absolute error of at most 2^-10 below 2^-6 (subnormal
spacing 2^-9); the kernel divides by the fp32 sum of the unrounded p.  Its p
are taken against a running max m' no larger than the row's max m, so
p_j / l_kernel = w_j (the exact softmax weights) and l_kernel >= l =
exp(lse - m).  Hence, per element,

    |o - o_ref| <= |dv| (2^-4 sum_j w_j |v_j| + 2^-10 sum_j |v_j| / l)
                   + ulp_bf16(o_ref) / 2 + slack,

with slack = 2^-10 |dv| sum_j w_j |v_j| + 1e-6 for the fp32 accumulations and
the approximate exp2 (each orders of magnitude below the rounding of P).  lse
uses only fp32 arithmetic and keeps the bf16 path's 1e-3.
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


def score_max_and_abs_v_sum(qf, kf, vf, s_eff, causal, rows):
    """Per sampled row: the max of its scaled, masked scores and, per column,
    the sum of |v_j| over its visible keys (both fp64)."""
    B, H, R = rows.shape
    N = kf.shape[2]
    m = np.empty((B, H, R))
    vs = np.empty((B, H, R, D))
    for b in range(B):
        for h in range(H):
            r = rows[b, h]
            s = s_eff * (qf[b, h, r].double() @ kf[b, h].double().T)
            cums = vf[b, h].double().abs().cumsum(0)
            if causal:
                s = s.masked_fill(torch.arange(N).view(1, N) > r.view(-1, 1), -math.inf)
                vs[b, h] = cums[r].numpy()
            else:
                vs[b, h] = cums[-1].expand(R, D).numpy()
            m[b, h] = s.max(dim=1).values.numpy()
    return m, vs


def check_fp8(q8, k8, v8, scale, causal, dq=1.0, dk=1.0, dv=1.0, rows=None):
    o, lse = run_fp8(q8, k8, v8, scale, causal, dq, dk, dv)
    B, H, N, _ = q8.shape
    if rows is None:
        rows = torch.arange(N, dtype=torch.int64).expand(B, H, N).contiguous()
    qf, kf, vf = (x.float() for x in (q8, k8, v8))  # exact
    s_eff = float(scale) * float(dq) * float(dk)
    o_ref, lse_ref = parity.oracle_reference(qf, kf, vf, s_eff, causal, rows)
    o_abs, _ = parity.oracle_reference(qf, kf, vf.abs(), s_eff, causal, rows)
    m, vsum = score_max_and_abs_v_sum(qf, kf, vf, s_eff, causal, rows)
    l_exact = np.exp(lse_ref - m)[..., None]
    o_ref = dv * o_ref
    o = parity.gather_rows(o, rows).float().numpy().astype(np.float64)
    lse = parity.gather_rows(lse, rows).numpy().astype(np.float64)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), "unwritten or non-finite output"
    err = np.abs(o - o_ref)
    main = abs(dv) * (2.0 ** -4 * o_abs + 2.0 ** -10 * vsum / l_exact)
    bound = main + parity.half_ulp_bf16(o_ref) + abs(dv) * 2.0 ** -10 * o_abs + 1e-6
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


def test_wide_scores_redo_blocks():
    # Q * 8 spreads the scores over tens of log2 units, so later blocks often
    # outgrow the running max by more than the E4M3 range allows and are redone
    q, k, v = e4m3_qkv(1, 4, 1024, seed=79, q_mult=8.0)
    check_fp8(q, k, v, 1 / math.sqrt(D), True)


@pytest.mark.parametrize("jump_at", [64, 320])
def test_score_jump(jump_at):
    # every query scores keys >= jump_at ~29 log2 units above the ones before
    # them: inside the first block it sets the exact max; in a later block it
    # forces a redo against that block's max and a rescale of O and l
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
