"""Build the oracle's shared library (test infrastructure only).

Compiles bq_oracle.c with gcc into liboracle_bq.so next to this file.  Plain
C11, FP64, no fused multiply-add contraction, OpenMP over rows.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bq_oracle.c")
OUT = os.path.join(HERE, "liboracle_bq.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(OUT)
            and os.path.getmtime(OUT) >= max(os.path.getmtime(SRC),
                                             os.path.getmtime(os.path.join(HERE, "bq_oracle.h")))):
        return OUT
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", OUT, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
