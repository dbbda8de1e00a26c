"""Compile the CPU oracle (``had_oracle.c``) into ``libhad_oracle.so``.

TEST INFRASTRUCTURE ONLY: the oracle is the reference the CUDA library is
checked against; nothing on the product path loads it.

Built with plain ``gcc -O2`` and OpenMP.  ``-ffast-math`` is deliberately
absent: the standardize step is an IEEE fp32 division with subnormals kept,
and fast-math would flush them.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "had_oracle.c")
LIB = os.path.join(HERE, "libhad_oracle.so")


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
           SRC, "-o", LIB + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
