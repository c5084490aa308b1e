"""Build libbitlinear.so (the sm_100a kernels and their C ABI) in-tree.

    python -m ternary_weight_bit_bitlinear_b200.build [--force]

nvcc cross-compiles for sm_100a on any host; no GPU is needed to build.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libbitlinear.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-Xptxas", "-warn-spills",
    "--expt-relaxed-constexpr",
    "-DBITLINEAR_BUILD",
]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
            if f.endswith((".cu", ".cuh"))] + [os.path.join(INCLUDE, "bitlinear.h")]


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/bitlinear.cu into libbitlinear.so unless it is up to date."""
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [NVCC, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-shared", "-cudart", "static",
           "-o", tmp, os.path.join(CSRC, "bitlinear.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
