"""B200 (sm_100a) exact attention forward: O = softmax(scale * Q K^T [causal]) V.

The compute runs in libfa_b200.so (hand-written CUDA for sm_100a behind the C
ABI in include/fa.h).  This module only marshals arguments to it: torch is
used for device memory and the current stream, nothing else.  There is no
fallback: if the library is missing or the GPU is not an sm_100 part, calls
raise.

    import tiled_exact_attention_fa_b200 as fa
    o, lse = fa.forward(q, k, v, causal=True)      # q, k, v: [B, H, N, d]
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa_b200.so")

FA_DTYPE_F32 = 0
FA_DTYPE_BF16 = 1
FA_OK = 0
FA_ERR_INVALID_ARGUMENT = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_CUDA = 3
FA_ERR_DEVICE_TIMEOUT = 4

# Every entry point of include/*.h with its ctypes signature.
_SIGNATURES = {
    "fa_fwd": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 4 +
               [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "fa_fwd_noalloc": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 4 +
                       [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "fa_fwd_fp8": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 4 +
                   [ctypes.c_float] * 4 + [ctypes.c_int, ctypes.c_void_p]),
    "fa_fwd_host": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 4 +
                    [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "fa_fwd_fp8_host": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 4 +
                        [ctypes.c_float] * 4 + [ctypes.c_int, ctypes.c_void_p]),
    "fa_decode": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 5 +
                  [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "fa_decode_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64] * 5),
    "fa_bwd": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int64] * 4 +
               [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "fa_bwd_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64] * 4),
    "fa_merge": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "fa_check_device_status": (ctypes.c_int, [ctypes.c_void_p]),
    "fa_fwd_kernel_choice": (ctypes.c_int, [ctypes.c_int64] * 4 + [ctypes.c_int] * 3 +
                             [ctypes.POINTER(ctypes.c_int)]),
    "fa_clock_record": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)]),
    "fa_noalloc_check_status": (ctypes.c_int, [ctypes.c_void_p]),
    "fa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fa_last_error": (ctypes.c_char_p, []),
    "fa_version": (ctypes.c_int, []),
    # include/fa_testing.h
    "fa_test_skip_one_arrival": (ctypes.c_int, []),
    "fa_test_force_forward_kernel": (ctypes.c_int, [ctypes.c_int]),
}

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, detail: str = ""):
        self.status = status
        msg = library().fa_status_string(status).decode()
        super().__init__(f"{msg}{': ' + detail if detail else ''}")


def library() -> ctypes.CDLL:
    """The loaded C-ABI library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m tiled_exact_attention_fa_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def version() -> int:
    return int(library().fa_version())


def _check(status: int):
    if status != FA_OK:
        raise FaError(status, library().fa_last_error().decode())


_DTYPES = {torch.bfloat16: FA_DTYPE_BF16, torch.float32: FA_DTYPE_F32}


def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, stream) -> int:
    """Direct C-ABI call with raw device pointers (ints); returns the status code."""
    return int(library().fa_fwd(q, k, v, o, lse, B, H, N, d, scale, int(causal), dtype, stream))


def forward_into(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                 lse: torch.Tensor, *, scale: float | None = None, causal: bool = False,
                 stream: torch.cuda.Stream | None = None) -> None:
    """Run the forward into caller-provided CUDA tensors o [B,H,N,d] and lse [B,H,N] fp32."""
    _check_qkv(q, k, v, o, lse)
    for t in (q, k, v, o, lse):
        if not t.is_cuda:
            raise ValueError("forward_into needs CUDA tensors")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    with torch.cuda.device(q.device):
        _check(fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      B, H, N, d, float(scale), causal, _DTYPES[q.dtype], s))


def _check_qkv(q, k, v, o, lse):
    if q.dtype not in _DTYPES or not (q.dtype == k.dtype == v.dtype == o.dtype):
        raise TypeError("q, k, v, o must all be bf16 or all fp32")
    if lse.dtype != torch.float32:
        raise TypeError("lse must be fp32")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape or o.shape != q.shape:
        raise ValueError("q, k, v, o must share one [B, H, N, d] shape")
    if lse.shape != q.shape[:3]:
        raise ValueError("lse must be [B, H, N]")
    for t in (q, k, v, o, lse):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def forward_fp8_into(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                     lse: torch.Tensor, *, descale_q: float = 1.0, descale_k: float = 1.0,
                     descale_v: float = 1.0, scale: float | None = None, causal: bool = False,
                     stream: torch.cuda.Stream | None = None) -> None:
    """fa_fwd_fp8: q, k, v torch.float8_e4m3fn [B, H, N, 128] tensors, each
    standing for its values times its descale factor; o bf16 [B, H, N, 128]
    and lse fp32 [B, H, N], caller-provided.  All CUDA tensors (asynchronous
    on `stream`), or all host tensors (fa_fwd_fp8_host: chunks of heads copied
    in, computed and copied out in a pipeline; valid once `stream` is
    synchronised)."""
    if not (q.dtype == k.dtype == v.dtype == torch.float8_e4m3fn):
        raise TypeError("q, k, v must be torch.float8_e4m3fn")
    if o.dtype != torch.bfloat16 or lse.dtype != torch.float32:
        raise TypeError("o must be bf16 and lse fp32")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape or o.shape != q.shape:
        raise ValueError("q, k, v, o must share one [B, H, N, d] shape")
    if lse.shape != q.shape[:3]:
        raise ValueError("lse must be [B, H, N]")
    on_device = [t.is_cuda for t in (q, k, v, o, lse)]
    if any(on_device) and not all(on_device):
        raise ValueError("forward_fp8_into takes all CUDA tensors or all host tensors")
    for t in (q, k, v, o, lse):
        if not t.is_contiguous():
            raise ValueError("forward_fp8_into needs contiguous tensors")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, float(scale),
            float(descale_q), float(descale_k), float(descale_v), int(causal))
    if all(on_device):
        s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
        with torch.cuda.device(q.device):
            _check(int(library().fa_fwd_fp8(*args, s)))
    else:
        # host tensors (pinned for asynchronous copies): fa_fwd_fp8_host on the
        # current device; o and lse are valid once `stream` is synchronised
        s = (stream or torch.cuda.current_stream()).cuda_stream
        _check(int(library().fa_fwd_fp8_host(*args, s)))


def forward_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, descale_q: float = 1.0,
                descale_k: float = 1.0, descale_v: float = 1.0, scale: float | None = None,
                causal: bool = False, stream: torch.cuda.Stream | None = None):
    """(o bf16, lse fp32) of the attention over E4M3 inputs (see forward_fp8_into).
    Host inputs give pinned host outputs that are complete when the call returns."""
    if q.is_cuda:
        o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    else:
        o = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True)
    forward_fp8_into(q, k, v, o, lse, descale_q=descale_q, descale_k=descale_k, descale_v=descale_v,
                     scale=scale, causal=causal, stream=stream)
    if not q.is_cuda:
        (stream or torch.cuda.current_stream()).synchronize()
    return o, lse


def forward_host_into(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                      lse: torch.Tensor, *, scale: float | None = None, causal: bool = False,
                      stream: torch.cuda.Stream | None = None) -> None:
    """fa_fwd_host on host tensors (pinned for asynchronous copies) on the
    current CUDA device; o and lse are valid once `stream` (default: the
    current stream) has been synchronised."""
    _check_qkv(q, k, v, o, lse)
    if any(t.is_cuda for t in (q, k, v, o, lse)):
        raise ValueError("forward_host_into takes host tensors")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = (stream or torch.cuda.current_stream()).cuda_stream
    _check(int(library().fa_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                     B, H, N, d, float(scale), int(causal), _DTYPES[q.dtype], s)))


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, scale: float | None = None,
            causal: bool = False, out: tuple[torch.Tensor, torch.Tensor] | None = None):
    """Exact attention forward.  Returns (o, lse).

    q, k, v: [B, H, N, d] bf16 or fp32, d in {64, 128}.  CUDA tensors give CUDA
    outputs.  Host tensors go through fa_fwd_host (chunks of heads copied in,
    computed and copied out in a pipeline on the current CUDA device) into
    host tensors -- `out=(o, lse)` if given, else new pinned tensors -- that
    are complete when the call returns.
    """
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    if not q.is_cuda:
        if out is None:
            out = (torch.empty(q.shape, dtype=q.dtype, pin_memory=True),
                   torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True))
        stream = torch.cuda.current_stream()
        forward_host_into(q, k, v, out[0], out[1], scale=scale, causal=causal, stream=stream)
        stream.synchronize()
        return out
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    forward_into(q, k, v, o, lse, scale=scale, causal=causal)
    if out is not None:
        out[0].copy_(o)
        out[1].copy_(lse)
        return out
    return o, lse


_decode_workspace: dict[int, torch.Tensor] = {}


def decode_workspace(B: int, H: int, Nq: int, Nk: int, d: int, device=None) -> torch.Tensor | None:
    """A device workspace large enough for fa_decode at these sizes, cached
    per device and grown when needed (None when none is needed)."""
    need = int(library().fa_decode_workspace_bytes(B, H, Nq, Nk, d))
    if need == 0:
        return None
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    ws = _decode_workspace.get(idx)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need + 256, dtype=torch.uint8, device=dev)
        _decode_workspace[idx] = ws
    return ws


def decode_into(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor, *,
                scale: float | None = None, causal: bool = False, workspace: torch.Tensor | None = None,
                stream: torch.cuda.Stream | None = None) -> None:
    """fa_decode into caller-provided CUDA tensors: q, o [B,H,Nq,d], k, v
    [B,H,Nk,d] (the cache), lse [B,H,Nq] fp32.  `workspace` defaults to a
    per-device cached one, so calls that may overlap on the GPU (different
    streams) must pass their own."""
    if q.dtype not in _DTYPES or not (q.dtype == k.dtype == v.dtype == o.dtype):
        raise TypeError("q, k, v, o must all be bf16 or all fp32")
    if lse.dtype != torch.float32:
        raise TypeError("lse must be fp32")
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape or o.shape != q.shape:
        raise ValueError("q, o must be [B, H, Nq, d] and k, v [B, H, Nk, d]")
    if q.shape[:2] != k.shape[:2] or q.shape[3] != k.shape[3] or lse.shape != q.shape[:3]:
        raise ValueError("inconsistent shapes")
    for t in (q, k, v, o, lse):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("decode_into needs contiguous CUDA tensors")
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(q.device):
        if workspace is None:
            workspace = decode_workspace(B, H, Nq, Nk, d, q.device)
        ptr, size = (0, 0) if workspace is None else (workspace.data_ptr(), workspace.numel() * workspace.element_size())
        if ptr % 256:
            off = 256 - ptr % 256
            ptr, size = ptr + off, size - off
        s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
        _check(int(library().fa_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                       B, H, Nq, Nk, d, float(scale), int(causal), _DTYPES[q.dtype],
                                       ptr or None, size, s)))


def decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, scale: float | None = None,
           causal: bool = False):
    """Attention of the new queries q [B,H,Nq,d] over the cache k, v
    [B,H,Nk,d] (CUDA tensors).  Returns (o, lse)."""
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    decode_into(q, k, v, o, lse, scale=scale, causal=causal)
    return o, lse


def backward_into(q, k, v, o, lse, dout, dq, dk, dv, *, scale: float | None = None, causal: bool = False,
                  workspace: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> None:
    """fa_bwd into caller-provided CUDA tensors (all [B, H, N, d] bf16, lse
    [B, H, N] fp32 as the forward wrote it)."""
    ts = (q, k, v, o, dout, dq, dk, dv)
    if any(t.dtype != torch.bfloat16 for t in ts) or lse.dtype != torch.float32:
        raise TypeError("the backward takes bf16 tensors and an fp32 lse")
    if any(t.shape != q.shape for t in ts) or q.dim() != 4 or lse.shape != q.shape[:3]:
        raise ValueError("all tensors must be [B, H, N, d], lse [B, H, N]")
    for t in ts + (lse,):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("backward_into needs contiguous CUDA tensors")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = int(library().fa_bwd_workspace_bytes(B, H, N, d))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
        _check(int(library().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                    dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                                    float(scale), int(causal), FA_DTYPE_BF16, workspace.data_ptr(),
                                    workspace.numel() * workspace.element_size(), s)))


def backward(q, k, v, o, lse, dout, *, scale: float | None = None, causal: bool = False):
    """Gradients (dq, dk, dv) of the forward for the upstream gradient dout."""
    q, k, v, o, dout = (t.contiguous() for t in (q, k, v, o, dout))
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    backward_into(q, k, v, o, lse.contiguous(), dout, dq, dk, dv, scale=scale, causal=causal)
    return dq, dk, dv


def merge(o_parts: torch.Tensor, lse_parts: torch.Tensor, *, stream: torch.cuda.Stream | None = None):
    """Combine results over disjoint key sets (fa_merge): o_parts [P, ..., d]
    and lse_parts [P, ...] CUDA tensors -> (o [..., d], lse [...])."""
    if o_parts.dtype not in _DTYPES or lse_parts.dtype != torch.float32:
        raise TypeError("o_parts must be bf16 or fp32 and lse_parts fp32")
    if lse_parts.shape != o_parts.shape[:-1] or not (o_parts.is_cuda and lse_parts.is_cuda):
        raise ValueError("o_parts [P, ..., d] and lse_parts [P, ...] on the GPU")
    o_parts, lse_parts = o_parts.contiguous(), lse_parts.contiguous()
    P, d = o_parts.shape[0], o_parts.shape[-1]
    rows = lse_parts[0].numel()
    o = torch.empty(o_parts.shape[1:], dtype=o_parts.dtype, device=o_parts.device)
    lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
    with torch.cuda.device(o_parts.device):
        s = (stream or torch.cuda.current_stream(o_parts.device)).cuda_stream
        _check(int(library().fa_merge(o_parts.data_ptr(), lse_parts.data_ptr(), P, rows, d, o.data_ptr(),
                                      lse.data_ptr(), _DTYPES[o_parts.dtype], s)))
    return o, lse


def check_device_status(stream: torch.cuda.Stream | None = None) -> None:
    """Synchronise and raise FaError(FA_ERR_DEVICE_TIMEOUT) if a kernel gave up on a wait."""
    s = (stream or torch.cuda.current_stream()).cuda_stream
    _check(int(library().fa_check_device_status(s)))


def forward_kernel_name(B: int, H: int, N: int, d: int, causal: bool, dtype=torch.bfloat16,
                        sm_count: int | None = None) -> str:
    """The kernel fa_fwd launches for this problem (fa_fwd_kernel_choice:
    bf16 takes whichever of the one-tile and two-tile kernels the library's
    schedule estimate finds faster; fp32 the CUDA-core kernel), for labels
    in bench lines and profiles.  sm_count None: the current device's."""
    out = ctypes.c_int(-1)
    _check(int(library().fa_fwd_kernel_choice(B, H, N, d, int(causal), _DTYPES[dtype], int(sm_count or 0),
                                               ctypes.byref(out))))
    c = str(bool(causal)).lower()
    return {0: f"fa_fwd_f32_kernel<{d},{c}>", 1: f"fa_fwd_bf16_kernel<{d},{c}>",
            2: f"fa_fwd_bf16_tile_kernel<{d},{c}>"}[out.value]


def clock_record(reset: bool = True, stream: torch.cuda.Stream | None = None) -> dict:
    """SM clock seen by the persistent forward kernels since the last reset
    (synchronises `stream`): summed CTA cycles and timer nanoseconds, the CTA
    count, the average clock in MHz and the cycles of an average CTA."""
    s = (stream or torch.cuda.current_stream()).cuda_stream
    out = (ctypes.c_int64 * 3)()
    _check(int(library().fa_clock_record(s, int(reset), out)))
    cycles, ns, ctas = int(out[0]), int(out[1]), int(out[2])
    return {"cycles": cycles, "ns": ns, "ctas": ctas,
            "sm_mhz": 1e3 * cycles / ns if ns else None,
            "cycles_per_cta": cycles / ctas if ctas else None}
