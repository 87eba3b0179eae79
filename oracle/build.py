"""Build the CPU oracle (plain C, gcc) into oracle/libfp8q_oracle.so.

Test infrastructure: the oracle is built so that the tests, the smoke check and the
benchmark's CPU-baseline leg can run it; the CUDA library never links it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fp8q_oracle.c")
LIB = os.path.join(HERE, "libfp8q_oracle.so")

# No fast-math and no FMA contraction: the SwiGLU spec is a sequence of individually
# rounded fp32 operations, and the rest is exact double/integer arithmetic.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp"
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
