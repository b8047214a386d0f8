"""Build the CPU oracle (plain C, gcc, OpenMP) into ``oracle/liboracle.so``.

Test infrastructure: the oracle is compiled with ``-O2 -ffp-contract=off`` and
without fast-math, so each float operation in it is a single IEEE-754
operation.  Building the checker is not using it; only the tests, the smoke
check and the benchmark's CPU baseline leg load the library.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cider_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
          "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra"]


def build_oracle(force: bool = False) -> str:
    """Compile the oracle if its library is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build_oracle(force=True))
