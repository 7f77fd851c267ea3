"""Builds libsigattn.so in-tree with nvcc for sm_100a (no GPU needed to build)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "sigattn_api.cu")
OUT = os.path.join(HERE, "libsigattn.so")
TRACE_OUT = os.path.join(HERE, "libsigattn_trace.so")   # diagnostic timeline build
DEPS = [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))] + [
    os.path.join(ROOT, "include", "sigattn.h")]


def nvcc_cmd(out: str = OUT, extra=()) -> list[str]:
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
            "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
            "-I", os.path.join(ROOT, "include"), SRC, "-o", out, *extra]


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    """Builds libsigattn.so, or with trace=True the diagnostic libsigattn_trace.so
    whose kernels record a timeline of one CTA (-DSIGATTN_TRACE)."""
    out = TRACE_OUT if trace else OUT
    stale = force or not os.path.exists(out) or any(
        os.path.getmtime(d) > os.path.getmtime(out) for d in DEPS)
    if stale:
        extra = ["-Xptxas", "-v"] if verbose else []
        if trace:
            extra.append("-DSIGATTN_TRACE")
        subprocess.run(nvcc_cmd(out=out, extra=extra), check=True)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv, trace="--trace" in sys.argv))
