"""Build the sm_100a CUDA library in place (nvcc; no GPU needed to compile)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libgdn_b200.so")
SOURCES = [os.path.join(HERE, "csrc", f) for f in
           ("gdn.cu", "device.cuh", "conv.cuh", "intra.cuh", "scan.cuh", "norm.cuh", "decode.cuh", "gemm.cuh", "cp.cuh",
            "fixup.cuh")]
HEADERS = [os.path.join(ROOT, "include", "gdn.h")]
NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-Xcompiler", "-fPIC", "-shared"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libgdn_b200.so next to this file if it is missing or out of date."""
    if force or stale(LIB, SOURCES + HEADERS):
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [nvcc(), *NVCC_FLAGS, "-I" + os.path.join(ROOT, "include"),
               "-o", tmp, os.path.join(HERE, "csrc", "gdn.cu")]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
