"""Work and traffic accounting for the attention forward (measurement helpers).

FLOPs follow the usual convention for the metric: two matrix products of
2*N*N*d multiply-adds each per head, 4*B*H*N^2*d in all, halved when the
causal mask removes the upper triangle.  (FlashAttention, Playable, EP 02
counts 2*N^2*d, which is the Q K^T product alone.)

Algorithmic bytes are the ideal traffic of a fused forward: Q, K and V read
once, O written once, and one fp32 log-sum-exp per row written once
(FlashAttention: Tiled & Fused, the diagram's "Output O written once").
The score matrix contributes nothing because it never leaves the chip.
"""
from __future__ import annotations


def attention_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def algorithmic_bytes(B: int, H: int, N: int, d: int, elem_bytes: int, lse_bytes: int = 4,
                      out_elem_bytes: int | None = None) -> int:
    """Q, K, V read once (elem_bytes each), O written once (out_elem_bytes,
    default elem_bytes) and one lse per row.  The E4M3 forward reads one-byte
    inputs and writes bf16: elem_bytes=1, out_elem_bytes=2."""
    rows = B * H * N
    out = elem_bytes if out_elem_bytes is None else out_elem_bytes
    return 3 * rows * d * elem_bytes + rows * d * out + rows * lse_bytes


def score_matrix_elements(N: int) -> int:
    """Entries of one head's N x N score matrix."""
    return N * N


def score_matrix_bytes(N: int, elem_bytes: int) -> int:
    """Bytes to hold one head's N x N score matrix in HBM."""
    return N * N * elem_bytes


def naive_score_round_trip_bytes(N: int, elem_bytes: int) -> int:
    """Write the score matrix to HBM and read it back once (per head)."""
    return 2 * N * N * elem_bytes


def ridge_intensity(peak_flops: float, bandwidth_bytes: float) -> float:
    """Arithmetic intensity (FLOP/byte) where compute and memory limits meet."""
    return peak_flops / bandwidth_bytes


def roofline_flops(intensity: float, peak_flops: float, bandwidth_bytes: float) -> float:
    """Attainable FLOP/s = min(peak compute, intensity x bandwidth)."""
    return min(peak_flops, intensity * bandwidth_bytes)
