"""Build libr2l.so in-tree with nvcc for sm_100a (B200).

The library is one translation unit (csrc/r2l.cu) linked against the static CUDA
runtime; the driver API (tensor-map encoding) is reached at run time through
cudaGetDriverEntryPoint, so the .so has no link-time dependency on libcuda.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
from typing import List, Optional

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libr2l.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libr2l.so")


def sources() -> List[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def build(force: bool = False, out: Optional[str] = None, extra: Optional[List[str]] = None, verbose: bool = False) -> str:
    out = out or LIB
    stale = force or not os.path.exists(out) or any(
        os.path.getmtime(s) > os.path.getmtime(out) for s in sources() + [os.path.join(INCLUDE, "r2l.h")])
    if not stale:
        return out
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-cudart", "static",
           "-I", INCLUDE, "-I", CSRC, "-o", out + ".tmp", os.path.join(CSRC, "r2l.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    cmd += list(extra or [])
    subprocess.check_call(cmd)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
