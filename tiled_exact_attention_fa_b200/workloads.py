"""Seeded synthetic workloads shared by the tests, the smoke check and the bench.

This module only generates inputs and picks sample rows; it holds none of the
attention arithmetic, and neither the oracle nor the CUDA path is imported
here.  The pages use no dataset: they speak of per-head N x d matrices Q, K, V
(Chapter 15 -- FlashAttention, "Standard vs Flash Attention") and give no
value distribution, so inputs are iid standard normal, drawn on the CPU from
one seeded torch generator in the order Q, K, V with shape [B, H, N, d] in
fp32, then cast to the workload's dtype.  The long-sequence workload scales Q
by 8 (a power of two, exact in bf16) to widen the score range so that the
online rescale is exercised.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: torch.dtype
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    q_mult: float = 1.0
    # rows per head checked against the oracle; None = every row
    sample_rows: int | None = None

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def dtype_name(self) -> str:
        return {torch.float32: "f32", torch.bfloat16: "bf16", torch.float8_e4m3fn: "e4m3"}[self.dtype]

    def describe(self) -> str:
        c = " causal" if self.causal else ""
        m = f" Q*{self.q_mult:g}" if self.q_mult != 1.0 else ""
        return f"{self.dtype_name} B={self.B} H={self.H} N={self.N} d={self.d}{c}{m} seed={self.seed}"


# The five workloads the build is measured and checked on.
WORKLOADS = [
    Workload("fp32_b1h1_n256_d64", torch.float32, 1, 1, 256, 64, False, 0),
    Workload("bf16_b1h8_n2048_d64", torch.bfloat16, 1, 8, 2048, 64, False, 1),
    Workload("bf16_b4h16_n4096_d128", torch.bfloat16, 4, 16, 4096, 128, False, 2, sample_rows=512),
    Workload("bf16_b2h32_n8192_d128_causal", torch.bfloat16, 2, 32, 8192, 128, True, 3, sample_rows=512),
    Workload("bf16_b1h16_n32768_d128_causal_q8", torch.bfloat16, 1, 16, 32768, 128, True, 4,
             q_mult=8.0, sample_rows=512),
]
# The E4M3 forward (fa_fwd_fp8) on the shapes of the two large bf16 workloads:
# the same fp32 draws, rounded to E4M3 (nearest; |x| < 448 for these draws, so
# nothing saturates), with descale factors 1.
FP8_WORKLOADS = [
    Workload("e4m3_b4h16_n4096_d128", torch.float8_e4m3fn, 4, 16, 4096, 128, False, 2, sample_rows=512),
    Workload("e4m3_b2h32_n8192_d128_causal", torch.float8_e4m3fn, 2, 32, 8192, 128, True, 3, sample_rows=512),
]
BY_NAME = {w.name: w for w in WORKLOADS + FP8_WORKLOADS}
HEADLINE = BY_NAME["bf16_b2h32_n8192_d128_causal"]


def make_inputs(w: Workload, device: str | torch.device = "cpu", pin: bool = False):
    """Q, K, V for workload ``w`` on ``device`` in ``w.dtype`` (seeded, CPU-drawn)."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.d)
    out = []
    for i in range(3):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if i == 0 and w.q_mult != 1.0:
            x.mul_(w.q_mult)
        x = x.to(w.dtype)
        if pin:
            x = x.pin_memory()
        out.append(x.to(device) if str(device) != "cpu" else x)
    return tuple(out)


def random_qkv(B, H, N, d, dtype, seed, q_mult=1.0, device="cpu"):
    """Ad-hoc shapes for edge-case tests, drawn the same way as the workloads."""
    w = Workload("adhoc", dtype, B, H, N, d, False, seed, q_mult=q_mult)
    return make_inputs(w, device=device)


def sample_rows(w: Workload, per_head: int | None = None):
    """Row indices [B, H, R] checked against the oracle.

    Every row when the workload checks all rows; otherwise, per (b, h), a
    seeded random permutation's first ``per_head`` rows together with the tile
    boundary rows {0, 127, 128, N-1}, padded to one common count R with further
    rows of the same permutation, and sorted.
    """
    per_head = per_head if per_head is not None else w.sample_rows
    if per_head is None or per_head >= w.N:
        return torch.arange(w.N, dtype=torch.int64).expand(w.B, w.H, w.N).contiguous()
    forced = sorted({r for r in (0, 127, 128, w.N - 1) if 0 <= r < w.N})
    R = min(w.N, per_head + len(forced))
    out = torch.empty((w.B, w.H, R), dtype=torch.int64)
    for b in range(w.B):
        for h in range(w.H):
            g = torch.Generator(device="cpu").manual_seed(w.seed * 1_000_003 + b * w.H + h)
            perm = torch.randperm(w.N, generator=g)
            chosen = list(forced)
            seen = set(chosen)
            for r in perm.tolist():
                if len(chosen) >= R:
                    break
                if r not in seen:
                    chosen.append(r)
                    seen.add(r)
            out[b, h] = torch.tensor(sorted(chosen), dtype=torch.int64)
    return out


# ------------------------------------------------------------------ decode
# A generation step over a key/value cache ("FlashAttention: Tiled & Fused",
# card "KV Cache: Why Generation Speeds Up"): nq new queries per head over a
# cache of nk positions whose last nq rows are the new tokens' own keys and
# values.  Same recipe: iid standard normal, drawn Q, K, V in that order.

@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    dtype: torch.dtype
    B: int
    H: int
    nq: int
    nk: int
    d: int
    causal: bool
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def cache_bytes(self) -> int:
        """K and V of the cache: what one step must read from HBM."""
        return 2 * self.B * self.H * self.nk * self.d * (2 if self.dtype == torch.bfloat16 else 4)


DECODE_WORKLOADS = [
    # a batch of 16 sequences of 16k cached tokens, 32 heads: 4.3 GB of cache per step
    DecodeWorkload("bf16_decode_b16h32_q1_nk16384_d128", torch.bfloat16, 16, 32, 1, 16384, 128, True, 5),
    # one long sequence, 8 heads, 256k cached tokens: split-KV over ~150 chunks per head
    DecodeWorkload("bf16_decode_b1h8_q1_nk262144_d128", torch.bfloat16, 1, 8, 1, 262144, 128, True, 6),
    # four new tokens at once (speculative / chunked step), causal among them
    DecodeWorkload("bf16_decode_b8h32_q4_nk32768_d128", torch.bfloat16, 8, 32, 4, 32768, 128, True, 7),
    # the same with a batch of 2 (1.07 GB of cache)
    DecodeWorkload("bf16_decode_b2h32_q4_nk32768_d128", torch.bfloat16, 2, 32, 4, 32768, 128, True, 8),
]
DECODE_BY_NAME = {w.name: w for w in DECODE_WORKLOADS}
DECODE_HEADLINE = DECODE_BY_NAME["bf16_decode_b16h32_q1_nk16384_d128"]


def make_decode_inputs(w: DecodeWorkload, device: str | torch.device = "cpu", pin: bool = False):
    """q [B,H,nq,d], k, v [B,H,nk,d] for decode workload ``w`` (seeded, CPU-drawn:
    Q, then K, then V, each as B consecutive draws of one batch element's
    [H, n, d] in fp32, cast to the workload's dtype)."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    out = []
    for n in (w.nq, w.nk, w.nk):
        x = torch.empty((w.B, w.H, n, w.d), dtype=w.dtype, pin_memory=pin)
        for b in range(w.B):
            x[b] = torch.randn((w.H, n, w.d), generator=g, dtype=torch.float32).to(w.dtype)
        out.append(x.to(device) if str(device) != "cpu" else x)
    return tuple(out)
