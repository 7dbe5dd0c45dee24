"""Build the test-only tcgen05 layout probe (libumma_probe.so) with nvcc."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "umma_probe.cu")
LIB = os.path.join(HERE, "libumma_probe.so")
ROOT = os.path.join(HERE, "..", "..")
DEPS = [SRC, os.path.join(ROOT, "hybrid_linear_attention_mixer_b200", "csrc", "device.cuh"),
        os.path.join(ROOT, "include", "gdn.h")]


def build(force=False):
    if force or not os.path.exists(LIB) or any(os.path.getmtime(d) > os.path.getmtime(LIB) for d in DEPS):
        nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.check_call([nvcc if os.path.exists(nvcc) else "nvcc", "-O2", "-std=c++17",
                               "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                               "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include"), "-o", tmp, SRC])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
