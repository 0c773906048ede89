"""Build libmoe.so (the CUDA library) in-tree with nvcc for sm_100a."""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoe.so")
LIB_CHECKS = os.path.join(PKG, "libmoe_checks.so")  # every row index range-checked
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["metadata.cu", "permute.cu", "gemm.cu", "moe.cu", "noalloc.cu", "backward.cu", "selftest.cu",
           "ep.cu"]
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-shared", "--threads", "4",
]


def _inputs():
    return [os.path.join(CSRC, s) for s in SOURCES] + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(INCLUDE, "moe.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose_ptxas: bool = False, checks: bool = False) -> str:
    """Compile libmoe.so, or with checks=True the range-checked libmoe_checks.so."""
    lib = LIB_CHECKS if checks else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [NVCC] + FLAGS + ["-I", INCLUDE, "-I", CSRC, "-o", lib] + \
        (["-DMOE_CHECKS=1"] if checks else []) + [os.path.join(CSRC, s) for s in SOURCES]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv,
                checks="--checks" in sys.argv))
