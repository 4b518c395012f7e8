"""Build the C-ABI shared library libfa_b200.so in-tree with nvcc (sm_100a).

    python -m tiled_exact_attention_fa_b200.build [--verbose-ptxas]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the CUDA driver's tensor-map encoder through the runtime's
driver entry-point query, so it loads on a machine without a GPU.
"""
from __future__ import annotations

import argparse
import hashlib
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libfa_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
SOURCES = ["fa_api.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC", "-cudart", "static",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is needed to build libfa_b200.so")


def _inputs_digest() -> str:
    h = hashlib.sha1()
    for d in (CSRC, INCLUDE):
        for name in sorted(os.listdir(d)):
            if name.endswith((".cu", ".cuh", ".h")):
                with open(os.path.join(d, name), "rb") as f:
                    h.update(name.encode() + f.read())
    h.update(" ".join(ARCH + FLAGS).encode())
    return h.hexdigest()


_TOKENS = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"|\'(?:\\.|[^\'\\])*\'', re.S)


def code_digest(files=None) -> str:
    """Digest of the library's code (or of the given csrc files) with comments
    and layout removed: it changes when the compiled code can change, not
    when a comment does."""
    h = hashlib.sha1()
    if files is None:
        paths = [os.path.join(d, n) for d in (CSRC, INCLUDE) for n in sorted(os.listdir(d))
                 if n.endswith((".cu", ".cuh", ".h"))]
    else:
        paths = [os.path.join(CSRC, n) for n in files]
    for path in paths:
        with open(path) as f:
            text = _TOKENS.sub(lambda m: " " if m.group(0)[0] == "/" else m.group(0), f.read())
        h.update(os.path.basename(path).encode() + " ".join(text.split()).encode())
    h.update(" ".join(ARCH + FLAGS).encode())
    return h.hexdigest()


# the sources each kernel is compiled from (for records tied to one kernel)
KERNEL_SOURCES = {
    "forward": ["fa_fwd_tc.cuh", "sm100_ptx.cuh"],
    "forward_tile": ["fa_fwd_tc1.cuh", "fa_fwd_tc.cuh", "sm100_ptx.cuh"],
    "decode": ["fa_decode.cuh", "sm100_ptx.cuh"],
    "decode_mma": ["fa_decode_mma.cuh", "fa_decode.cuh", "sm100_ptx.cuh"],
    "forward_fp8": ["fa_fwd_fp8_tc.cuh", "fa_fwd_tc.cuh", "sm100_ptx.cuh"],
    "backward": ["fa_bwd_tc.cuh", "fa_fwd_tc.cuh", "sm100_ptx.cuh"],
}


def is_current() -> bool:
    stamp = LIB_PATH + ".sha1"
    return os.path.exists(LIB_PATH) and os.path.exists(stamp) and open(stamp).read().strip() == _inputs_digest()


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Compile libfa_b200.so next to this file; skip when sources are unchanged."""
    if not force and not verbose_ptxas and is_current():
        return LIB_PATH
    cmd = [nvcc(), *ARCH, *FLAGS, f"-I{INCLUDE}", f"-I{CSRC}"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    tmp = f"{LIB_PATH}.{os.getpid()}.tmp"
    cmd += [os.path.join(CSRC, s) for s in SOURCES] + ["-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    with open(LIB_PATH + ".sha1", "w") as f:
        f.write(_inputs_digest() + "\n")
    return LIB_PATH


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true", help="print registers/spills per kernel")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))
    sys.exit(0)
