"""Build the CSA2 CPU oracle (test infrastructure) into oracle/libcsa2_oracle.so.

Plain gcc, double precision, no fast-math and no FMA contraction, so that every
operation rounds exactly as written in csa2_oracle.c. OpenMP only parallelises over
independent outputs.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csa2_oracle.c")
OUT = os.path.join(HERE, "libcsa2_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= os.path.getmtime(SRC):
        return OUT
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-fvisibility=hidden", "-Wall", "-o", OUT + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
