"""Build the CPU oracle shared library (plain C, gcc).

Test infrastructure: the library built here is loaded only by the tests, the
smoke check and the CPU-baseline leg of the benchmark.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qlinear_oracle.c")
LIB = os.path.join(HERE, "libqlinear_oracle.so")

# -ffp-contract=off and no fast-math keep every float32 step a single IEEE
# operation with round-to-nearest-even (no FMA contraction, no reassociation).
CFLAGS = ["-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fno-fast-math",
          "-fexcess-precision=standard", "-fopenmp", "-fPIC", "-shared", "-Wall"]


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", *CFLAGS, SRC, "-o", LIB, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
