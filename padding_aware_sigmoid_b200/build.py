"""Builds libsigattn.so in-tree with nvcc for sm_100a (no GPU needed to build)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "sigattn_api.cu")
OUT = os.path.join(HERE, "libsigattn.so")
DEPS = [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))] + [
    os.path.join(ROOT, "include", "sigattn.h")]


def nvcc_cmd(out: str = OUT, extra=()) -> list[str]:
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
            "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
            "-I", os.path.join(ROOT, "include"), SRC, "-o", out, *extra]


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds libsigattn.so when it is missing or older than its sources."""
    stale = force or not os.path.exists(OUT) or any(
        os.path.getmtime(d) > os.path.getmtime(OUT) for d in DEPS)
    if stale:
        extra = ["-Xptxas", "-v"] if verbose else []
        subprocess.run(nvcc_cmd(out=OUT, extra=extra), check=True)
    return OUT


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
