"""Build the CUDA library ``libhad.so`` in-tree for sm_100a (B200).

``nvcc`` cross-compiles without a GPU.  The library links the CUDA runtime
statically, so it only needs the driver at run time.  Fast-math is off on
purpose: the standardize step relies on IEEE division with subnormals.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libhad.so")
SOURCES = ["had_api.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _newest_input():
    paths = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    paths += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= _newest_input()):
        return LIB
    cmd = (["nvcc"] + ARCH +
           ["-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
            "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
            "-I", INCLUDE, "-I", CSRC, "-o", LIB + ".tmp"] +
           (["-Xptxas", "-v"] if verbose else []) +
           [os.path.join(CSRC, s) for s in SOURCES])
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
