"""Builds libsparse_attn.so in-tree for sm_100a with nvcc (no GPU needed).

    python -m dynamic_block_sparse_fractal_b200.build
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIBDIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIBDIR, "libsparse_attn.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + [os.path.join(HERE, "..", "include", "sparse_attn.h"), __file__]
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in deps)


TRACE_LIB = os.path.join(LIBDIR, "libsparse_attn_trace.so")


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    """The library; with trace=True a separate diagnostics build whose
    attention kernel records a timeline of one CTA (see trace_attn.py)."""
    lib = TRACE_LIB if trace else LIB
    if not force and up_to_date(lib):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-Xptxas", "-v" if verbose else "-O3", *(["-DSA_TRACE=1"] if trace else []),
           "-o", tmp, *sources()]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                trace="--trace" in sys.argv))
