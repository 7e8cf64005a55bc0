"""Build the sm_100a CUDA library libmla_b200.so in-tree with nvcc.

The library is one translation unit (csrc/mla_abi.cu and the headers it
includes), linked with the static CUDA runtime so that it depends on no
libcuda at load time; the driver entry points it needs are fetched at run
time through the runtime API.
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "mla_abi.cu")
LIB = os.path.join(PKG, "libmla_b200.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def _sources():
    return glob.glob(os.path.join(PKG, "csrc", "*")) + [os.path.join(ROOT, "include", "mla.h")]


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in _sources())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-o", LIB, SRC]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
