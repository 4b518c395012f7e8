"""fp64 CPU oracle for the exact attention forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product path (the CUDA
library and its Python binding) never imports, links or calls it, and this
package imports nothing from the product.

The oracle is the plain definition of attention as the pages state standard
attention (Chapter 15 -- FlashAttention, "Standard vs Flash Attention": S =
Q K^T, P = softmax(S), O = P V), with the scale and causal mask applied in the
plainest way and the per-row log-sum-exp in natural log.  The arithmetic lives
in ``fa_oracle.c`` (plain C, fp64, OpenMP over heads and row blocks); this
module only compiles it with gcc and marshals numpy arrays.

Pins (see tests/test_oracle_*.py): closed forms (Q = 0, a single key, causal
row 0), invariances (key permutation, future-key independence, softmax shift,
affine V), the online-softmax ledger of the pages (FlashAttention, Playable,
EP 04), torch's fp64 math attention as a library cross-check, hand-worked tiny
cases, and source mutants that each of those must catch.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import platform
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fa_oracle.c")
# x86-64-v3 (AVX2 + FMA) keeps the build portable across the hosts the tests
# run on; no tuning flags beyond -O3 and OpenMP.
CFLAGS = ["-O3", "-march=x86-64-v3", "-fopenmp", "-shared", "-fPIC", "-std=c11"]

_lib = None


def _lib_path(src: str = _SRC) -> str:
    with open(src, "rb") as f:
        digest = hashlib.sha1(f.read() + " ".join(CFLAGS).encode()).hexdigest()[:12]
    return os.path.join(_HERE, "_build", f"libfa_oracle_{platform.machine()}_{digest}.so")


def build(src: str = _SRC, out: str | None = None, extra_flags=()) -> str:
    """Compile ``src`` with gcc into a shared library; returns its path.

    ``src``/``out``/``extra_flags`` let the mutation tests compile altered
    copies of the oracle into a temporary directory.
    """
    out = out or _lib_path(src)
    if os.path.exists(out):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = f"{out}.{os.getpid()}.tmp"
    subprocess.run(["gcc", *CFLAGS, *extra_flags, src, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, out)
    return out


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    f = lib.oracle_attention_fwd
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64,
        ctypes.c_void_p, ctypes.c_void_p]
    g = lib.oracle_attention_decode
    g.restype = ctypes.c_int
    g.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 4 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    b = lib.oracle_attention_bwd
    b.restype = ctypes.c_int
    b.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    br = lib.oracle_attention_bwd_rows
    br.restype = ctypes.c_int
    br.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    m = lib.oracle_lse_merge
    m.restype = ctypes.c_int
    m.argtypes = [ctypes.c_void_p] * 2 + [ctypes.c_int64] * 3 + [ctypes.c_void_p] * 2
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_version.restype = ctypes.c_int
    return lib


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the oracle library (building it first if needed)."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(load().oracle_num_threads())


def attention_fwd(q, k, v, scale: float, causal: bool, rows=None, lib=None):
    """Exact attention forward in fp64.

    q, k, v: arrays of shape [B, H, N, d] holding the exact input values
        (fp32, or anything numpy converts to fp32 without rounding, e.g. the
        fp32 upcast of bf16 data).
    rows: None for every query row, else an int array [B, H, R] of row indices
        (the same count R for every head).
    Returns (o, lse): o is [B, H, R, d] fp64, lse is [B, H, R] fp64 natural log.
    """
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    if q.ndim != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, H, N, d] shape")
    B, H, N, d = q.shape
    if rows is None:
        rows = np.broadcast_to(np.arange(N, dtype=np.int64), (B, H, N))
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if rows.ndim != 3 or rows.shape[:2] != (B, H):
        raise ValueError("rows must be [B, H, R]")
    R = rows.shape[2]
    o = np.empty((B, H, R, d), dtype=np.float64)
    lse = np.empty((B, H, R), dtype=np.float64)
    rc = lib.oracle_attention_fwd(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, B * H, N, d, float(scale),
        int(bool(causal)), rows.ctypes.data, R, o.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_attention_fwd failed with code {rc}")
    return o, lse


def attention_decode(q, k, v, scale: float, causal: bool, lib=None):
    """Attention of nq new queries over nk cached keys, in fp64.

    q: [B, H, nq, d]; k, v: [B, H, nk, d] (exact input values, fp32).  Query i
    sits at position nk - nq + i; causal restricts it to keys <= that position.
    Returns (o, lse): o is [B, H, nq, d] fp64, lse is [B, H, nq] fp64 natural log.
    """
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    if q.ndim != 4 or k.ndim != 4 or k.shape != v.shape or q.shape[:2] != k.shape[:2] or q.shape[3] != k.shape[3]:
        raise ValueError("q must be [B, H, nq, d] and k, v [B, H, nk, d]")
    B, H, nq, d = q.shape
    nk = k.shape[2]
    o = np.empty((B, H, nq, d), dtype=np.float64)
    lse = np.empty((B, H, nq), dtype=np.float64)
    rc = lib.oracle_attention_decode(q.ctypes.data, k.ctypes.data, v.ctypes.data, B * H, nq, nk, d,
                                     float(scale), int(bool(causal)), o.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_attention_decode failed with code {rc}")
    return o, lse


def attention_bwd(q, k, v, do, scale: float, causal: bool, lib=None):
    """Gradients (dq, dk, dv) of the attention output with respect to q, k, v
    for the upstream gradient `do`, in fp64.  All inputs [B, H, N, d] (exact
    values, fp32); returns three [B, H, N, d] fp64 arrays."""
    lib = lib or load()
    q, k, v, do = (np.ascontiguousarray(x, dtype=np.float32) for x in (q, k, v, do))
    if q.ndim != 4 or not (q.shape == k.shape == v.shape == do.shape):
        raise ValueError("q, k, v, do must share one [B, H, N, d] shape")
    B, H, N, d = q.shape
    dq, dk, dv = (np.empty((B, H, N, d), dtype=np.float64) for _ in range(3))
    rc = lib.oracle_attention_bwd(q.ctypes.data, k.ctypes.data, v.ctypes.data, do.ctypes.data, B * H, N, d,
                                  float(scale), int(bool(causal)), dq.ctypes.data, dk.ctypes.data, dv.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_attention_bwd failed with code {rc}")
    return dq, dk, dv


def attention_bwd_rows(q, k, v, do, scale: float, causal: bool, qrows, krows, lib=None):
    """The gradients of attention_bwd for chosen rows only, in fp64, for heads
    too long for the n x n matrices.

    q, k, v, do: [B, H, N, d] (exact input values, fp32).  qrows [B, H, nq]
    and krows [B, H, nk]: int row indices per head.  Returns (dq [B, H, nq, d]
    for the query rows, dk, dv [B, H, nk, d] for the key rows), fp64.
    """
    lib = lib or load()
    q, k, v, do = (np.ascontiguousarray(x, dtype=np.float32) for x in (q, k, v, do))
    if q.ndim != 4 or not (q.shape == k.shape == v.shape == do.shape):
        raise ValueError("q, k, v, do must share one [B, H, N, d] shape")
    B, H, N, d = q.shape
    qrows = np.ascontiguousarray(qrows, dtype=np.int64)
    krows = np.ascontiguousarray(krows, dtype=np.int64)
    if qrows.ndim != 3 or qrows.shape[:2] != (B, H) or krows.ndim != 3 or krows.shape[:2] != (B, H):
        raise ValueError("qrows and krows must be [B, H, count]")
    nq, nk = qrows.shape[2], krows.shape[2]
    dq = np.empty((B, H, nq, d), dtype=np.float64)
    dk, dv = (np.empty((B, H, nk, d), dtype=np.float64) for _ in range(2))
    rc = lib.oracle_attention_bwd_rows(q.ctypes.data, k.ctypes.data, v.ctypes.data, do.ctypes.data, B * H, N, d,
                                       float(scale), int(bool(causal)), qrows.ctypes.data, nq, krows.ctypes.data,
                                       nk, dq.ctypes.data, dk.ctypes.data, dv.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_attention_bwd_rows failed with code {rc}")
    return dq, dk, dv


def lse_merge(o_parts, lse_parts, lib=None):
    """Combine per-key-set results: o_parts [P, ..., d], lse_parts [P, ...]
    (same leading shape) -> (o, lse) over the union of the key sets, fp64."""
    lib = lib or load()
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float32)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float32)
    P = o_parts.shape[0]
    lead = o_parts.shape[1:-1]
    d = o_parts.shape[-1]
    if lse_parts.shape != (P,) + lead:
        raise ValueError("lse_parts must match o_parts without its last axis")
    rows = int(np.prod(lead)) if lead else 1
    o = np.empty(lead + (d,), dtype=np.float64)
    lse = np.empty(lead, dtype=np.float64)
    rc = lib.oracle_lse_merge(o_parts.ctypes.data, lse_parts.ctypes.data, P, rows, d, o.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_lse_merge failed with code {rc}")
    return o, lse
