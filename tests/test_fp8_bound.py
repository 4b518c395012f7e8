"""The E4M3 error bound (tests/fp8_bound.py) on the CPU: a numpy model of
the kernel's arithmetic (blocks of 128 keys, running max moved only on jumps
above 8 log2 units, p rounded to E4M3 as the P V operand, l over the
unrounded p, O times descale_v) stays inside it, and plausible mistakes in
that arithmetic land outside it -- so the GPU test's bound is neither
violated by the intended rounding nor loose enough to hide an error."""
import math

import numpy as np
import pytest
import torch

from tiled_exact_attention_fa_b200 import workloads as W
from tests import fp8_bound

D = 128
LOG2E = 1.4426950408889634


def round_to(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x)).float().to(dtype).double().numpy()


def model(q8, k8, v8, scale, causal, dq=1.0, dk=1.0, dv=1.0, p_dtype=torch.float8_e4m3fn,
          use_descale_qk=True, use_dv=True, mask_shift=0, rescale_o=True, slack=8.0):
    """The kernel's steps in fp64 (exact scores), with switches for mistakes."""
    qf, kf, vf = (x.double().numpy() for x in (q8, k8, v8))
    B, H, N, _ = qf.shape
    with np.errstate(invalid="ignore", divide="ignore"):
        return _model(qf, kf, vf, scale, causal, dq, dk, dv, p_dtype, use_descale_qk, use_dv, mask_shift,
                      rescale_o, slack)


def _model(qf, kf, vf, scale, causal, dq, dk, dv, p_dtype, use_descale_qk, use_dv, mask_shift, rescale_o, slack):
    B, H, N, _ = qf.shape
    sl = scale * (dq * dk if use_descale_qk else 1.0) * LOG2E
    out = np.zeros((B, H, N, D))
    rows = np.arange(N)
    for b in range(B):
        for h in range(H):
            s = (qf[b, h] @ kf[b, h].T) * sl
            if causal:
                s = np.where(np.arange(N)[None, :] <= rows[:, None] + mask_shift, s, -np.inf)
            m = np.full(N, -np.inf)
            l = np.zeros(N)
            o = np.zeros((N, D))
            for j0 in range(0, N, 128):
                blk = s[:, j0:j0 + 128]
                bm = blk.max(axis=1)
                move = (bm > m + slack) | ((m == -np.inf) & (bm > -np.inf))
                alpha = np.where(move & (m > -np.inf), np.exp2(np.where(move, m - bm, 0.0)), 1.0)
                alpha = np.where(move & (m == -np.inf), 0.0, alpha)
                l *= alpha
                if rescale_o:
                    o *= alpha[:, None]
                m = np.where(move, bm, m)
                neg = np.where(m == -np.inf, 0.0, -m)
                p = np.exp2(blk + neg[:, None])
                l += p.sum(axis=1)
                o += round_to(p, p_dtype) @ vf[b, h, j0:j0 + 128]
            out[b, h] = (dv if use_dv else 1.0) * o / l[:, None]
    return out


def fits(o, o_ref, bound):
    return bool((np.abs(o - o_ref) <= bound).all())


CASES = [
    # B, H, N, causal, q_mult, dq, dk, dv, scale sign
    (1, 2, 300, True, 1.0, 1.0, 1.0, 1.0, 1),
    (1, 2, 300, False, 1.0, 1.0, 1.0, 1.0, 1),
    (1, 2, 384, True, 1.0, 0.5, 3.0, -0.25, 1),
    (1, 2, 260, True, 8.0, 1.0, 1.0, 1.0, 1),   # wide scores: the max moves
    (1, 1, 200, True, 1.0, 1.0, 1.0, 1.0, -1),  # negative scale
]


@pytest.mark.parametrize("B,H,N,causal,q_mult,dq,dk,dv,sign", CASES)
def test_model_of_the_kernel_is_inside_the_bound(B, H, N, causal, q_mult, dq, dk, dv, sign):
    q, k, v = W.random_qkv(B, H, N, D, torch.float8_e4m3fn, seed=N + 17, q_mult=q_mult)
    scale = sign / math.sqrt(D)
    o_ref, _, bound = fp8_bound.reference(q, k, v, scale, causal, dq, dk, dv)
    o = model(q, k, v, scale, causal, dq, dk, dv)
    err = np.abs(o - o_ref)
    assert (err <= bound).all(), float((err / bound).max())
    # and the bound is not vacuous: the model's rounding uses a real share of it
    assert (err / bound).max() > 0.05


def test_bound_catches_mistakes():
    q, k, v = W.random_qkv(1, 2, 300, D, torch.float8_e4m3fn, seed=5)
    qw, kw, vw = W.random_qkv(1, 2, 260, D, torch.float8_e4m3fn, seed=6, q_mult=8.0)
    scale = 1 / math.sqrt(D)
    ref = fp8_bound.reference(q, k, v, scale, True, 0.5, 3.0, 0.5)
    refw = fp8_bound.reference(qw, kw, vw, scale, True)
    o_ref, _, bound = ref
    assert fits(model(q, k, v, scale, True, 0.5, 3.0, 0.5), o_ref, bound)
    # P rounded to E5M2 (two mantissa bits) instead of E4M3
    assert not fits(model(q, k, v, scale, True, 0.5, 3.0, 0.5, p_dtype=torch.float8_e5m2), o_ref, bound)
    # descale_v not applied
    assert not fits(model(q, k, v, scale, True, 0.5, 3.0, 0.5, use_dv=False), o_ref, bound)
    # descale_q * descale_k left out of the scores' scale
    assert not fits(model(q, k, v, scale, True, 0.5, 3.0, 0.5, use_descale_qk=False), o_ref, bound)
    # causal mask off by one (a row misses its own key, or sees the next one);
    # row 0 is left out of the first, where it would have no key at all
    o_m = model(q, k, v, scale, True, 0.5, 3.0, 0.5, mask_shift=-1)
    assert not fits(o_m[:, :, 1:], o_ref[:, :, 1:], bound[:, :, 1:])
    assert not fits(model(q, k, v, scale, True, 0.5, 3.0, 0.5, mask_shift=1), o_ref, bound)
    # the running max moves but O is not rescaled (wide scores make it move)
    o_refw, _, boundw = refw
    assert fits(model(qw, kw, vw, scale, True), o_refw, boundw)
    assert not fits(model(qw, kw, vw, scale, True, rescale_o=False), o_refw, boundw)
