"""Build libssa.so (the C-ABI library of include/ssa.h) in-tree with nvcc for sm_100a."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = [os.path.join(HERE, "csrc", "ssa_fwd.cu"), os.path.join(HERE, "csrc", "ssa_decode.cu")]
DEPS = SRC + [os.path.join(HERE, "csrc", "ptx.cuh"), os.path.join(HERE, "csrc", "internal.h"),
              os.path.join(ROOT, "include", "ssa.h")]
LIB = os.path.join(HERE, "libssa.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build(force: bool = False, verbose: bool = False) -> str:
    stale = not os.path.exists(LIB) or any(os.path.getmtime(d) > os.path.getmtime(LIB) for d in DEPS)
    if force or stale:
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
               "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
               "-o", LIB + ".tmp"] + SRC
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
