"""Build the in-tree CUDA library ``libsdq.so`` for sm_100a.

    python swiglu_backward_int8_b200/build.py [--verbose]

(run it as a script: importing the package needs the library it builds)

nvcc compiles ``csrc/sdq_api.cu`` (host API + the fused kernel) and
``csrc/fwd_api.cu`` (the forward-side SwiGLU + q8_1 kernel) into a shared
library with a C ABI (``include/sdq.h``); the CUDA runtime is linked
statically and the driver's tensor-map encoder is looked up at run time, so
the library needs only the NVIDIA driver at load time.
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
LIB = os.path.join(PKG, "libsdq.so")
SOURCES = [os.path.join(CSRC, f) for f in ("sdq_api.cu", "fwd_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("sdq_kernel.cuh", "sdq_ptx.cuh", "fwd_kernel.cuh")] + [
    os.path.join(INCLUDE, "sdq.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC,-O2",
              "-shared", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libsdq.so if it is missing or older than its sources."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(f) for f in DEPS)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), *SOURCES, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
