"""Compile libzero_b200.so in-tree for sm_100a (nvcc; static CUDA runtime)."""
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "libzero_b200.so")
SOURCES = [os.path.join(PKG, "csrc", f) for f in ("api.cpp", "kernels.cu", "noalloc.cu", "zero3.cpp", "zero3_gather.cu")]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared"]


def build(verbose: bool = False) -> str:
    cmd = ["nvcc", *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(PKG, "csrc"), "-o", LIB_PATH, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    return LIB_PATH


if __name__ == "__main__":
    build(verbose=True)
