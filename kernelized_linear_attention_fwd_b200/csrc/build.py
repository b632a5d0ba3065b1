"""Builds libkata.so (the C-ABI library) for sm_100a with nvcc.

    python kernelized_linear_attention_fwd_b200/csrc/build.py [--verbose]

The shared object lands in the package directory beside the Python binding.
Cross-compiles without a GPU.  `--verbose` adds -Xptxas -v (registers, spills,
shared memory per kernel).
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
OUT = os.path.join(PKG, "libkata.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(HERE, "*.cuh"))) + [os.path.join(ROOT, "include", "kata.h")]


def up_to_date():
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(f) <= t for f in sources() + headers() + [__file__])


def build(force=False, verbose=False):
    if not force and not verbose and up_to_date():
        return OUT
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = OUT + ".tmp%d" % os.getpid()
    cmd = [nvcc] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose else []) + sources() + ["-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
