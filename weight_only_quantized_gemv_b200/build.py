"""Build the in-tree shared library ``libqlinear.so`` for sm_100a with nvcc.

The library is a plain C ABI (``include/qlinear.h``) with the CUDA runtime linked
statically, so loading it needs no GPU; only the first CUDA call does.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqlinear.so")

SOURCES = ["qlinear.cu", "dequant.cu", "prefill_tc.cu", "codebook.cu", "policy.cpp", "pack.cpp"]
HEADERS = ["kernels.cuh", "layout.h", "policy.h", "dequant_frag.cuh"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, ptxas_verbose: bool = False) -> list:
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-shared", "-cudart", "static", "-Xcompiler", "-fPIC,-fopenmp",
           "-I", INCLUDE, "-I", CSRC]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    cmd += ["-o", out, "-lgomp", "-ldl"]
    return cmd


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "qlinear.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if any source is newer than it; return its path."""
    if force or _stale(LIB):
        tmp = LIB + ".tmp"
        cmd = command(tmp, ptxas_verbose=verbose)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
        if verbose:
            sys.stderr.write(r.stdout + r.stderr)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
