"""fa_bwd against the fp64 backward oracle.

The workload definition states no tolerance for gradients; the bound here
follows from the arithmetic: inputs and outputs are bf16 (relative rounding
2^-9), P and dS are rounded to bf16 before the tensor-core products
(another 2^-9 each) and everything else accumulates in fp32.  Each gradient
is held to max-abs error <= 2e-2 * max|ref| + half a bf16 ulp of the exact
value, and mean-abs error <= 2e-3 * max|ref|, per tensor; and, as a whole, to
a relative L2 error <= 5e-3: three independent bf16 roundings of relative
RMS 2^-9 / sqrt(3) each (P, dS, the output) give about 2e-3, and the bound
leaves a factor 2.5 for the fp32 accumulation order and for the correlation
of the roundings.  Sizes up to the full 8192-token headline shape, where the
row-sampled oracle checks dq on sampled query rows and dk, dv on sampled key
rows."""
import math

import numpy as np
import pytest
import torch

import oracle
import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build
from tests.parity import half_ulp_bf16

pytestmark = pytest.mark.gpu


def make(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return tuple(torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(4))


def check(got: torch.Tensor, ref: np.ndarray, name: str):
    x = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(x).all(), name
    err = np.abs(x - ref)
    scale = np.abs(ref).max()
    beyond = err - half_ulp_bf16(ref)
    assert beyond.max() <= 2e-2 * scale, (name, float(beyond.max()), float(scale))
    assert err.mean() <= 2e-3 * scale, (name, float(err.mean()), float(scale))
    rel2 = float(np.linalg.norm(x - ref) / np.linalg.norm(ref))
    assert rel2 <= 5e-3, (name, rel2)
    return float(err.max() / scale)


@pytest.mark.parametrize("B,H,N,d,causal", [
    (1, 2, 128, 128, False),
    (1, 2, 256, 128, True),
    (2, 1, 300, 128, True),     # ragged last block
    (1, 3, 517, 64, False),
    (1, 1, 640, 64, True),
    (1, 2, 1000, 128, False),
    (2, 5, 384, 128, True),     # heads in two launch groups (8 + 2)
    (1, 2, 1000, 64, True),     # ragged, many query blocks per key block
])
def test_backward_matches_oracle(B, H, N, d, causal):
    fa_build.build()
    q, k, v, do = make(B, H, N, d, seed=N + d)
    scale = 1.0 / math.sqrt(d)
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    o = torch.empty_like(qc)
    lse = torch.empty(q.shape[:3], device="cuda")
    fa.forward_into(qc, kc, vc, o, lse, scale=scale, causal=causal)
    dq, dk, dv = fa.backward(qc, kc, vc, o, lse, doc, scale=scale, causal=causal)
    torch.cuda.synchronize()
    fa.check_device_status()
    rq, rk, rv = oracle.attention_bwd(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                      do.float().numpy(), scale, causal)
    for got, ref, name in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check(got, ref, name)


def test_backward_invariants_at_a_larger_size():
    # properties that hold at any size: the key gradients of a head sum to
    # zero and the value gradients sum to the sum of dO (up to bf16 rounding)
    fa_build.build()
    B, H, N, d = 1, 4, 4096, 128
    q, k, v, do = (t.cuda() for t in make(B, H, N, d, seed=5))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device="cuda")
    fa.forward_into(q, k, v, o, lse, causal=True)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    fa.check_device_status()
    sk = dk.float().sum(dim=2)
    sv, sdo = dv.float().sum(dim=2), do.float().sum(dim=2)
    assert sk.abs().max().item() <= 2e-2 * dk.float().abs().max().item() * math.sqrt(N)
    assert (sv - sdo).abs().max().item() <= 1e-2 * sdo.abs().max().item() + 0.5


def _sample_rows(N, count, seed):
    g = np.random.default_rng(seed)
    forced = np.array([0, 127, 128, N - 1])
    rest = g.choice(np.setdiff1d(np.arange(N), forced), count, replace=False)
    return np.sort(np.r_[forced, rest])


def _check_sampled(q, k, v, do, dq, dk, dv, scale, causal, heads, seed):
    """dq on sampled query rows and dk, dv on sampled key rows of the given
    (b, h) heads, against the row-sampled fp64 oracle."""
    for (b, h) in heads:
        sl = lambda t: t[b:b + 1, h:h + 1].float().cpu().numpy()
        rows = _sample_rows(q.shape[2], 60, seed + 7 * b + h)[None, None]
        rq, rk, rv = oracle.attention_bwd_rows(sl(q), sl(k), sl(v), sl(do), scale, causal, rows, rows)
        take = lambda t: torch.from_numpy(np.take_along_axis(sl(t), rows[..., None], axis=2))
        for got, ref, name in ((take(dq), rq, "dq"), (take(dk), rk, "dk"), (take(dv), rv, "dv")):
            check(got, ref, f"{name} head {(b, h)}")


def test_backward_headline_shape_sampled_rows():
    # the workload and launch `bench.py --path backward` times: B2 H32 N8192
    # d128 causal, seed 3; two heads checked on sampled rows
    from tiled_exact_attention_fa_b200 import workloads as W
    fa_build.build()
    w = W.HEADLINE
    q, k, v = (t.cuda() for t in W.make_inputs(w))
    g = torch.Generator().manual_seed(w.seed + 1000)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16).cuda()
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device="cuda")
    fa.forward_into(q, k, v, o, lse, scale=w.scale, causal=w.causal)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    fa.check_device_status()
    _check_sampled(q, k, v, do, dq, dk, dv, w.scale, w.causal, [(0, 0), (1, 31)], seed=w.seed)


def test_backward_full_length_not_causal():
    fa_build.build()
    B, H, N, d = 1, 2, 8192, 128
    q, k, v, do = (t.cuda() for t in make(B, H, N, d, seed=8192))
    scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device="cuda")
    fa.forward_into(q, k, v, o, lse, scale=scale, causal=False)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, scale=scale, causal=False)
    torch.cuda.synchronize()
    fa.check_device_status()
    _check_sampled(q, k, v, do, dq, dk, dv, scale, False, [(0, 0), (0, 1)], seed=11)
