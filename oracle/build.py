"""Build the CPU oracle library ``oracle/libcsa2_ref.so`` with gcc.

Test infrastructure only: the oracle is loaded by the test suite, the smoke
check and the benchmark's CPU-baseline leg, never by the CUDA library.

The flags keep every floating-point step as written: no fast-math and no
contraction of a*b+c into a fused multiply-add, so the fp32 quantisation steps
are IEEE binary32 operations in the order the source states them.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csa2_ref.c")
LIB = os.path.join(HERE, "libcsa2_ref.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
          "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
