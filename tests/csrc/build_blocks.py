"""Builds tests/csrc/libtcgen05_blocks.so (test-only kernels) for sm_100a."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
SRC = os.path.join(HERE, "tcgen05_blocks.cu")
OUT = os.path.join(HERE, "libtcgen05_blocks.so")
DEPS = [SRC, os.path.join(ROOT, "kernelized_linear_attention_fwd_b200", "csrc", "sm100.cuh"),
        os.path.join(ROOT, "kernelized_linear_attention_fwd_b200", "csrc", "tmap.cuh")]


def build(force=False):
    if not force and os.path.exists(OUT) and all(
            os.path.getmtime(d) <= os.path.getmtime(OUT) for d in DEPS):
        return OUT
    tmp = OUT + ".tmp%d" % os.getpid()
    subprocess.check_call([os.environ.get("NVCC", "nvcc"), "-gencode",
                           "arch=compute_100a,code=sm_100a", "-lineinfo", "-O2", "-std=c++17",
                           "-Xcompiler", "-fPIC", "-shared", SRC, "-o", tmp])
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force=True))
