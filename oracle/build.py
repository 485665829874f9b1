"""Compile the CPU oracle (fftconv_oracle.c) into oracle/liboracle.so.

Test infrastructure: only the tests, ``__graft_entry__`` and bench.py's CPU
baseline leg use the oracle.  Plain gcc, fp64, no fast-math and no FMA
contraction, so the oracle's arithmetic is exactly what its source says.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fftconv_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
          "-D_DEFAULT_SOURCE", "-shared", "-fPIC", "-Wall", "-Wextra"]


def build(force: bool = False, src: str = SRC, out: str = LIB, extra=()) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", *CFLAGS, *extra, src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
