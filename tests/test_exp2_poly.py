"""The polynomial 2^x used for part of the softmax exponentials.

CPU: the constants in sm100_ptx.cuh are the ones the committed Remez fit
produces, and the routine's fp32 steps (emulated with numpy float32) stay
within the fit's relative error bound, far below bf16's half-ulp (2^-9) that P
is rounded to.  GPU: the device routine against CUDA's exp2f (torch.exp2).
"""
import os
import re
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tiled_exact_attention_fa_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly  # noqa: E402

BOUND = 8e-5  # the fit's 7.5e-5 plus fp32 evaluation rounding


def header_constants():
    text = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    vals = {}
    for k in range(4):
        m = re.search(rf"kExp2C{k}\s*=\s*([0-9a-fx.p+-]+)f;", text)
        vals[k] = float.fromhex(m.group(1))
    return [vals[k] for k in range(4)]


def emulate(x):
    """exp2_poly2's steps in numpy float32, in the kernel's order."""
    c0, c1, c2, c3 = (np.float32(c) for c in header_constants())
    magic = np.float32(12582912.0)
    x = np.minimum(np.maximum(np.asarray(x, np.float32), np.float32(-125.0)), np.float32(127.0))
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)  # exact (Sterbenz), as the fused form is

    def fma(a, b, c):  # one rounding to fp32 of a*b + c (the product is exact in fp64)
        return (np.float64(a) * b.astype(np.float64) + np.float64(c)).astype(np.float32) \
            if np.isscalar(a) else (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)

    p = fma(c3, f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_constants_come_from_the_fit():
    coeffs, err = fit_exp2_poly.fit()
    assert err < 7.6e-5
    for got, want in zip(header_constants(), np.asarray(coeffs, np.float32)):
        assert got == float(want)


def test_emulated_relative_error():
    x = np.linspace(-120.0, 8.0, 2_000_001).astype(np.float32)
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < BOUND, rel.max()
    # integers are hit at f = 0: close to, but not exactly, a power of two
    assert np.all(np.abs(emulate(np.arange(-100, 8, dtype=np.float32)) /
                         np.exp2(np.arange(-100, 8)) - 1) < BOUND)


def test_clamp_below_range():
    y = emulate(np.array([-126.0, -1000.0, -np.inf], np.float32))
    assert np.all(y > 0) and np.all(y < 2.0 ** -124)


def test_clamp_above_range():
    # values the softmax must see as "far too large" (so that the block is
    # redone against its exact max): finite, at least 2^126, never wrapped
    with np.errstate(over="ignore"):
        y = emulate(np.array([126.6, 127.0, 127.6, 128.0, 200.0, 1e30, np.inf], np.float32))
    assert np.all(np.isfinite(y)) and np.all(y >= 2.0 ** 126), y


@pytest.mark.gpu
def test_device_routine_against_cuda_exp2():
    import tiled_exact_attention_fa_b200 as fa
    from tiled_exact_attention_fa_b200 import build as fb
    fb.build()
    x = torch.linspace(-120.0, 8.0, 1_000_001, device="cuda", dtype=torch.float32)
    x = torch.cat([x, torch.tensor([127.0, 128.0, 200.0, float("inf"), -1000.0, float("-inf")], device="cuda")])
    y = torch.empty_like(x)
    rc = fa.library().fa_test_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel(),
                                          torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    ref = torch.exp2(x[:-6])  # CUDA's exp2f
    rel = (y[:-6].double() / ref.double() - 1).abs().max().item()
    assert rel < BOUND, rel
    tail = y[-6:].cpu()
    assert torch.isfinite(tail).all() and (tail[:4] >= 2.0 ** 126).all() and (tail[4:] > 0).all()
    # and the device result matches the float32 emulation of the same steps
    # (fp64-then-fp32 rounding of the fused steps can differ by one ulp on ties)
    got = y.cpu().numpy().view(np.int32).astype(np.int64)
    want = emulate(x.cpu().numpy()).view(np.int32).astype(np.int64)
    assert np.abs(got - want).max() <= 1
    assert np.mean(got == want) > 0.999
