"""The C-ABI boundary on the CPU: the library loads without a GPU, exports every
entry point include/fa.h declares, and rejects bad arguments before making
any CUDA call (so these run, and must pass, on a machine with no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import tiled_exact_attention_fa_b200 as fa
from tiled_exact_attention_fa_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in os.listdir(os.path.join(ROOT, "include")) if h.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.library()


def declared_functions():
    names = []
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(fa_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fa_fwd", "fa_check_device_status", "fa_status_string", "fa_last_error", "fa_version"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\S+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        getattr(lib, name)  # and ctypes can resolve it


def test_binding_covers_every_entry_point():
    assert set(declared_functions()) == set(fa._SIGNATURES)


def test_version(lib):
    assert fa.version() == 10000


def test_status_strings(lib):
    for code in range(0, 5):
        s = lib.fa_status_string(code).decode()
        assert s.startswith(("FA_OK", "FA_ERR_"))
    assert "unknown" in lib.fa_status_string(99).decode()


# Fake, never-dereferenced addresses: every case below must be rejected by
# the argument checks, which run before any CUDA call.
A = 0x10000000
NB = 1 << 24  # spacing between the fake buffers


def call(lib, q=A, k=A + NB, v=A + 2 * NB, o=A + 3 * NB, lse=A + 4 * NB, B=1, H=1, N=128, d=128,
         scale=0.1, causal=0, dtype=fa.FA_DTYPE_BF16, entry="fa_fwd"):
    return getattr(lib, entry)(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, None)


@pytest.mark.parametrize("kwargs,code", [
    (dict(q=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(k=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(v=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(o=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(lse=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(B=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(H=-1), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(N=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(d=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(dtype=7), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(q=A + 8), fa.FA_ERR_INVALID_ARGUMENT),          # misaligned
    (dict(o=A + 3 * NB + 2), fa.FA_ERR_INVALID_ARGUMENT),  # misaligned
    (dict(lse=A + 4 * NB + 2), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(o=A + 16), fa.FA_ERR_INVALID_ARGUMENT),          # o overlaps q
    (dict(lse=A + 3 * NB + 64), fa.FA_ERR_INVALID_ARGUMENT),  # lse inside o
    (dict(N=(1 << 30) + 1), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(B=1 << 20, H=1 << 20), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),
])
@pytest.mark.parametrize("entry", ["fa_fwd", "fa_fwd_noalloc"])
def test_rejected_before_cuda(lib, kwargs, code, entry):
    # fa_fwd_noalloc runs the same checks, also before any CUDA call
    assert call(lib, entry=entry, **kwargs) == code
    assert lib.fa_last_error().decode() != ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_no_gpu_is_an_error_not_a_fallback(lib):
    # well-formed arguments on a machine without a GPU: a CUDA error, never a result
    assert call(lib) == fa.FA_ERR_CUDA
    assert call(lib, entry="fa_fwd_noalloc") == fa.FA_ERR_CUDA
    assert lib.fa_noalloc_check_status(None) == fa.FA_ERR_CUDA
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises((RuntimeError, AssertionError)):
        fa.forward(q, q, q)


def call_host(lib, q=A, k=A + NB, v=A + 2 * NB, o=A + 3 * NB, lse=A + 4 * NB, B=1, H=1, N=128, d=128,
              scale=0.1, causal=0, dtype=fa.FA_DTYPE_BF16):
    return lib.fa_fwd_host(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, None)


@pytest.mark.parametrize("kwargs,code", [
    (dict(q=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(lse=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(N=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(dtype=7), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(o=A + 16), fa.FA_ERR_INVALID_ARGUMENT),          # o overlaps q
    (dict(lse=A + 3 * NB + 64), fa.FA_ERR_INVALID_ARGUMENT),  # lse inside o
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
])
def test_host_entry_rejected_before_cuda(lib, kwargs, code):
    assert call_host(lib, **kwargs) == code
    assert lib.fa_last_error().decode() != ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_host_entry_needs_no_alignment_but_a_gpu(lib):
    # host buffers need no alignment: a misaligned q passes the checks and the
    # call then fails on the missing GPU
    assert call_host(lib, q=A + 2) == fa.FA_ERR_CUDA


def call_decode(lib, q=A, k=A + NB, v=A + 2 * NB, o=A + 3 * NB, lse=A + 4 * NB, B=1, H=1, Nq=1, Nk=128, d=128,
                scale=0.1, causal=0, dtype=fa.FA_DTYPE_BF16, ws=A + 6 * NB, ws_bytes=1 << 20):
    return lib.fa_decode(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, ws, ws_bytes, None)


@pytest.mark.parametrize("kwargs,code", [
    (dict(q=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(v=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(Nq=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(Nk=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(Nq=5, Nk=4, causal=1), fa.FA_ERR_INVALID_ARGUMENT),  # causal queries must fit in the cache
    (dict(dtype=3), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(k=A + NB + 4), fa.FA_ERR_INVALID_ARGUMENT),         # misaligned
    (dict(o=A + 64), fa.FA_ERR_INVALID_ARGUMENT),             # o overlaps q
    (dict(Nk=1 << 20, ws=0), fa.FA_ERR_INVALID_ARGUMENT),     # a workspace is needed and missing
    (dict(Nk=1 << 20, ws_bytes=16), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(Nk=1 << 20, ws=A + 6 * NB + 16), fa.FA_ERR_INVALID_ARGUMENT),  # workspace not 256-byte aligned
    (dict(d=80), fa.FA_ERR_UNSUPPORTED),
])
def test_decode_rejected_before_cuda(lib, kwargs, code):
    assert call_decode(lib, **kwargs) == code
    assert lib.fa_last_error().decode() != ""


def test_decode_workspace_size(lib):
    # one CTA per head already fills the GPU: no workspace
    assert lib.fa_decode_workspace_bytes(64, 32, 1, 4096, 128) == 0
    # a single long head is split into chunks: partials (m, l, O) per chunk + counters
    one = lib.fa_decode_workspace_bytes(1, 1, 1, 1 << 20, 128)
    assert one > 0 and one % 256 == 0
    assert lib.fa_decode_workspace_bytes(1, 1, 8, 1 << 20, 128) > one  # partials per query
    assert lib.fa_decode_workspace_bytes(0, 1, 1, 10, 128) == 0       # invalid sizes


def test_backward_rejected_before_cuda(lib):
    args = [A, A + NB, A + 2 * NB, A + 3 * NB, A + 4 * NB, A + 5 * NB, A + 6 * NB, A + 7 * NB, A + 8 * NB]
    ok = dict(B=1, H=1, N=128, d=128, scale=0.1, causal=0, dtype=fa.FA_DTYPE_BF16, ws=A + 9 * NB, wsb=1 << 20)

    def bwd(args, B=1, H=1, N=128, d=128, scale=0.1, causal=0, dtype=fa.FA_DTYPE_BF16, ws=A + 9 * NB, wsb=1 << 20):
        return lib.fa_bwd(*args, B, H, N, d, scale, causal, dtype, ws, wsb, None)

    assert bwd([0] + args[1:]) == fa.FA_ERR_INVALID_ARGUMENT          # null q
    assert bwd(args, N=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert bwd(args, dtype=fa.FA_DTYPE_F32) == fa.FA_ERR_UNSUPPORTED   # bf16 only
    assert bwd(args, d=96) == fa.FA_ERR_UNSUPPORTED
    assert bwd(args, ws=0) == fa.FA_ERR_INVALID_ARGUMENT               # workspace missing
    assert bwd(args, wsb=4) == fa.FA_ERR_INVALID_ARGUMENT              # workspace too small
    assert bwd(args[:6] + [A + 16] + args[7:]) == fa.FA_ERR_INVALID_ARGUMENT  # dq overlaps q
    assert bwd(args[:6] + [A + 6 * NB + 8] + args[7:]) == fa.FA_ERR_INVALID_ARGUMENT  # misaligned
    assert lib.fa_bwd_workspace_bytes(2, 3, 1000, 128) >= 2 * 3 * 1000 * 4
    assert lib.fa_bwd_workspace_bytes(0, 3, 1000, 128) == 0


def test_merge_rejected_before_cuda(lib):
    def merge(op=A, lp=A + NB, parts=2, rows=10, d=128, o=A + 2 * NB, lse=A + 3 * NB, dtype=fa.FA_DTYPE_BF16):
        return lib.fa_merge(op, lp, parts, rows, d, o, lse, dtype, None)

    assert merge(op=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert merge(parts=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert merge(rows=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert merge(dtype=5) == fa.FA_ERR_INVALID_ARGUMENT
    assert merge(d=32) == fa.FA_ERR_UNSUPPORTED
    assert merge(o=A + 2 * NB + 4) == fa.FA_ERR_INVALID_ARGUMENT   # misaligned
    assert merge(o=A + 64) == fa.FA_ERR_INVALID_ARGUMENT           # output inside the parts
    assert lib.fa_last_error().decode() != ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_other_entries_need_a_gpu(lib):
    # well-formed calls of the other entry points fail with a CUDA error on a
    # machine without a GPU: never a CPU result
    assert lib.fa_decode(A, A + NB, A + 2 * NB, A + 3 * NB, A + 4 * NB, 1, 1, 1, 128, 128, 0.1, 0,
                         fa.FA_DTYPE_BF16, None, 0, None) == fa.FA_ERR_CUDA
    assert lib.fa_merge(A, A + NB, 2, 10, 128, A + 2 * NB, A + 3 * NB, fa.FA_DTYPE_BF16, None) == fa.FA_ERR_CUDA
    ws = lib.fa_bwd_workspace_bytes(1, 1, 128, 128)
    assert lib.fa_bwd(A, A + NB, A + 2 * NB, A + 3 * NB, A + 4 * NB, A + 5 * NB, A + 6 * NB, A + 7 * NB,
                      A + 8 * NB, 1, 1, 128, 128, 0.1, 0, fa.FA_DTYPE_BF16, A + 9 * NB, ws, None) == fa.FA_ERR_CUDA


def call_fp8(lib, q=A, k=A + NB, v=A + 2 * NB, o=A + 3 * NB, lse=A + 4 * NB, B=1, H=1, N=128, d=128,
             scale=0.1, dq=1.0, dk=1.0, dv=1.0, causal=0):
    return lib.fa_fwd_fp8(q, k, v, o, lse, B, H, N, d, scale, dq, dk, dv, causal, None)


@pytest.mark.parametrize("kwargs,code", [
    (dict(q=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(lse=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(N=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(dq=float("inf")), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(dv=float("nan")), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(scale=1e30, dq=1e30, dk=1e30), fa.FA_ERR_INVALID_ARGUMENT),  # product overflows fp32
    (dict(q=A + 8), fa.FA_ERR_INVALID_ARGUMENT),                       # misaligned
    (dict(o=A + 2 * NB - 64), fa.FA_ERR_INVALID_ARGUMENT),             # bf16 o (2 bytes/elem) reaches v
    (dict(lse=A + 3 * NB + 64), fa.FA_ERR_INVALID_ARGUMENT),           # lse inside o
    (dict(d=64), fa.FA_ERR_UNSUPPORTED),
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),
])
def test_fp8_rejected_before_cuda(lib, kwargs, code):
    assert call_fp8(lib, **kwargs) == code
    assert lib.fa_last_error().decode() != ""


def test_fp8_output_is_twice_the_input_bytes(lib):
    # o holds bf16: with q at A and o 16 KB below it, a 128 x 128 E4M3 head
    # (16 KB) ends at q's start but its bf16 output (32 KB) runs into q
    assert call_fp8(lib, o=A - 16384) == fa.FA_ERR_INVALID_ARGUMENT


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_fp8_needs_a_gpu(lib):
    assert call_fp8(lib) == fa.FA_ERR_CUDA


def test_force_forward_kernel_hook(lib):
    # the test hook only records the choice: no CUDA call, so it runs here
    for bad in (3, -1, 99):
        assert lib.fa_test_force_forward_kernel(bad) == fa.FA_ERR_INVALID_ARGUMENT
        assert "0, 1 or 2" in lib.fa_last_error().decode()
    for ok in (1, 2, 0):
        assert lib.fa_test_force_forward_kernel(ok) == fa.FA_OK


def test_clock_record_arguments(lib):
    assert lib.fa_clock_record(None, 0, None) == fa.FA_ERR_INVALID_ARGUMENT
    if not torch.cuda.is_available():
        out = (ctypes.c_int64 * 3)()
        assert lib.fa_clock_record(None, 1, out) == fa.FA_ERR_CUDA


def test_forward_kernel_name_follows_the_size_rule():
    # fa_fwd_kernel_choice with a given SM count makes no CUDA call.  Cases
    # whose faster kernel was measured on a B200 (148 SMs), both masks:
    name = fa.forward_kernel_name
    tile, two = "fa_fwd_bf16_tile_kernel", "fa_fwd_bf16_kernel"
    assert name(1, 8, 2048, 64, False, sm_count=148) == tile + "<64,false>"   # 128 tiles: one wave
    assert name(1, 16, 2048, 128, True, sm_count=148) == tile + "<128,true>"  # 256 tiles, causal: 0.71x
    assert name(1, 8, 4096, 128, True, sm_count=148) == tile + "<128,true>"   # 0.63x
    assert name(1, 16, 2048, 128, False, sm_count=148) == two + "<128,false>"  # 256 tiles, no mask: 1.10x
    assert name(1, 16, 4096, 128, True, sm_count=148) == two + "<128,true>"    # 512 tiles, causal: 1.13x
    assert name(2, 32, 8192, 128, True, sm_count=148) == two + "<128,true>"    # headline, beyond 8 per SM
    assert name(1, 1, 256, 64, False, torch.float32, sm_count=148) == "fa_fwd_f32_kernel<64,false>"
    # the choice follows the SM count it is given
    assert name(1, 16, 2048, 128, False, sm_count=512) == tile + "<128,false>"


def test_kernel_choice_arguments(lib):
    out = ctypes.c_int(-1)
    assert lib.fa_fwd_kernel_choice(1, 1, 128, 128, 0, fa.FA_DTYPE_BF16, 148, None) == fa.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_fwd_kernel_choice(0, 1, 128, 128, 0, fa.FA_DTYPE_BF16, 148, ctypes.byref(out)) == \
        fa.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_fwd_kernel_choice(1, 1, 128, 80, 0, fa.FA_DTYPE_BF16, 148, ctypes.byref(out)) == \
        fa.FA_ERR_UNSUPPORTED
    if not torch.cuda.is_available():  # the current device's SM count needs a GPU
        assert lib.fa_fwd_kernel_choice(1, 1, 128, 128, 0, fa.FA_DTYPE_BF16, 0, ctypes.byref(out)) == fa.FA_ERR_CUDA


def call_fp8_host(lib, q=A, k=A + NB, v=A + 2 * NB, o=A + 3 * NB, lse=A + 4 * NB, B=1, H=1, N=128, d=128,
                  scale=0.1, dq=1.0, dk=1.0, dv=1.0, causal=0):
    return lib.fa_fwd_fp8_host(q, k, v, o, lse, B, H, N, d, scale, dq, dk, dv, causal, None)


@pytest.mark.parametrize("kwargs,code", [
    (dict(q=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(N=0), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(dq=float("inf")), fa.FA_ERR_INVALID_ARGUMENT),
    (dict(o=A + 2 * NB - 64), fa.FA_ERR_INVALID_ARGUMENT),   # bf16 o reaches v
    (dict(d=64), fa.FA_ERR_UNSUPPORTED),
])
def test_fp8_host_rejected_before_cuda(lib, kwargs, code):
    assert call_fp8_host(lib, **kwargs) == code


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_fp8_host_needs_no_alignment_but_a_gpu(lib):
    assert call_fp8_host(lib, q=A + 3) == fa.FA_ERR_CUDA


def test_c_program_uses_the_boundary(lib, tmp_path):
    # the headers compile as C99 and a C program links against the library
    # and calls it (the calls below make no CUDA call)
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_fa.c"
    src.write_text(
        '#include <stdio.h>\n#include "fa.h"\n#include "fa_testing.h"\n'
        "int main(void) {\n"
        "    int kernel = -1;\n"
        "    int rc = fa_fwd_kernel_choice(1, 8, 2048, 64, 0, FA_DTYPE_BF16, 148, &kernel);\n"
        "    int bad = fa_fwd(0, 0, 0, 0, 0, 1, 1, 1, 64, 0.1f, 0, FA_DTYPE_BF16, 0);\n"
        '    printf("%d %d %d %d %s\\n", fa_version(), rc, kernel, bad, fa_status_string(bad));\n'
        "    return 0;\n}\n")
    exe = tmp_path / "use_fa"
    pkg = os.path.dirname(fa.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", pkg, "-lfa_b200", "-Wl,-rpath," + pkg, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert out[:4] == [str(fa.version()), str(fa.FA_OK), "2", str(fa.FA_ERR_INVALID_ARGUMENT)]
    assert out[4].startswith("FA_ERR_INVALID_ARGUMENT")
