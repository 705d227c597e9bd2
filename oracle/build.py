"""Build the CPU oracle (plain C) into oracle/liboracle.so with gcc.

Test infrastructure only: the product library never links this.  Compiled
without fast-math and with -ffp-contract=off so that every float expression is
one IEEE operation in round-to-nearest-even.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "oracle.c")
    hdr = os.path.join(HERE, "oracle.h")
    if (not force and os.path.exists(SO)
            and os.path.getmtime(SO) >= max(os.path.getmtime(src), os.path.getmtime(hdr))):
        return SO
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-fno-finite-math-only", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", SO + ".tmp", src, "-lm"]
    subprocess.check_call(cmd)
    os.replace(SO + ".tmp", SO)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
