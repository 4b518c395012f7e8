"""Reference and error bound for the E4M3 forward (fa_fwd_fp8), shared by
the GPU parity tests and the CPU tests that check the bound itself.

The exact result is the pinned fp64 oracle's attention of the E4M3 values
(upcast exactly) with the scale scale * dq * dk, times dv.  The kernel's one
approximation is P rounded to E4M3 (round to nearest: relative error <= 2^-4
for normal values, absolute error <= 2^-10 below 2^-6), taken against a
running max no larger than the row max and normalised by the fp32 sum of the
unrounded p.  With w_j the exact softmax weights and l = exp(lse - max s):

    |o - o_ref| <= |dv| (2^-4 sum_j w_j |v_j| + 2^-10 sum_j |v_j| / l)
                   + ulp_bf16(o_ref) / 2 + 2^-10 |dv| sum_j w_j |v_j| + 1e-6

(the last two terms: the bf16 output and the fp32 accumulations / exp2).
"""
from __future__ import annotations

import math

import numpy as np
import torch

from tests import parity


def score_max_and_abs_v_sum(qf, kf, vf, s_eff, causal, rows):
    """Per sampled row: the max of its scaled, masked scores and, per column,
    the sum of |v_j| over its visible keys (both fp64)."""
    B, H, R = rows.shape
    N, d = kf.shape[2], kf.shape[3]
    m = np.empty((B, H, R))
    vs = np.empty((B, H, R, d))
    for b in range(B):
        for h in range(H):
            r = rows[b, h]
            s = s_eff * (qf[b, h, r].double() @ kf[b, h].double().T)
            cums = vf[b, h].double().abs().cumsum(0)
            if causal:
                s = s.masked_fill(torch.arange(N).view(1, N) > r.view(-1, 1), -math.inf)
                vs[b, h] = cums[r].numpy()
            else:
                vs[b, h] = cums[-1].expand(R, d).numpy()
            m[b, h] = s.max(dim=1).values.numpy()
    return m, vs


def reference(q8, k8, v8, scale, causal, dq=1.0, dk=1.0, dv=1.0, rows=None):
    """(o_ref, lse_ref, bound) for E4M3 inputs q8, k8, v8 (torch.float8_e4m3fn,
    CPU) at the given rows ([B, H, R] int64, None = all)."""
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
    main = abs(dv) * (2.0 ** -4 * o_abs + 2.0 ** -10 * vsum / l_exact)
    bound = main + parity.half_ulp_bf16(o_ref) + abs(dv) * 2.0 ** -10 * o_abs + 1e-6
    return o_ref, lse_ref, bound
