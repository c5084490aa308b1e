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


def units():
    """The translation units: the C ABI (bitlinear.cu) and one launcher unit
    per kernel family (launch_*.cu), compiled in parallel."""
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith(".cu")]


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every unit of csrc/ and link libbitlinear.so, unless it is up
    to date."""
    if not force and up_to_date():
        return LIB
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    procs, objs = [], []
    for src in units():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".%d.o" % os.getpid())
        cmd = [NVCC, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", "-o", obj, src]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd))
        procs.append((src, subprocess.Popen(cmd)))
        objs.append(obj)
    failed = [src for src, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc " + " ".join(failed))
    tmp = LIB + ".tmp.%d" % os.getpid()
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           "-cudart", "static", "-o", tmp, *objs])
    for obj in objs:
        os.remove(obj)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
