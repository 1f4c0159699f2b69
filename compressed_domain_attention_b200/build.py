"""Build ``libtq_b200.so`` (the C-ABI library, sm_100a kernels) in-tree with nvcc."""
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtq_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-ffp-contract=off",
    "-shared", "-cudart", "static",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + [
        os.path.join(HERE, "..", "include", "tq.h")]


def build_library(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in _inputs())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = [NVCC, *NVCC_FLAGS]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", LIB + ".tmp", *sources()]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build_library(force=True, verbose_ptxas="-v" in sys.argv))
