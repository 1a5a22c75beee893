"""Build the sm_100a CUDA library in-tree: ``fp8_quant_logscale_b200/libsdm_fp8.so``.

nvcc cross-compiles for sm_100a on a machine without a GPU.  The CUDA runtime
is linked statically, so the library needs only the NVIDIA driver at run time;
the driver's tensor-map encoder is reached through cudaGetDriverEntryPoint.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsdm_fp8.so")
SOURCES = ["api.cu", "quant.cu", "attention.cu", "attention_f16.cu", "prefill.cu"]
HEADERS = ["kernels.cuh", "ptx.cuh", "exp2_poly.cuh", "softmax.cuh", os.path.join("..", "..", "include", "sdm_fp8.h")]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsdm_fp8.so")
    return cand


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    return any(os.path.getmtime(f) > t for f in files)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ for sm_100a into libsdm_fp8.so (if stale)."""
    if not force and not _stale():
        return LIB
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH_FLAGS, "-lineinfo", "-Xcompiler", "-fPIC,-O3",
           "-shared", "-cudart", "static", "-o", LIB]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
