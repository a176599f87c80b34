"""Build step: compile libstepmoe.so in-tree for sm_100a (nvcc cross-compiles without a GPU)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libstepmoe.so")
SOURCES = ["api.cu", "route.cu", "permute.cu", "expert_ffn.cu", "combine.cu", "pack.cu", "noalloc.cu", "diag.cu", "fp8.cu", "selftest.cu"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-shared",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def build(verbose: bool = False, extra_flags=()) -> str:
    cmd = ["nvcc", *NVCC_FLAGS, *extra_flags, "-o", LIB, *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose=True)
