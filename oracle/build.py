"""Build the oracle's shared library (test infrastructure only).

The oracle is plain C99 in double precision, compiled with gcc and OpenMP over
independent (sequence, head) units.  It shares no source with the CUDA library.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kda_oracle.c")
LIB = os.path.join(HERE, "libkda_oracle.so")


def build(force: bool = False) -> str:
    """Compile oracle/libkda_oracle.so if it is missing or older than its sources."""
    srcs = [SRC, os.path.join(HERE, "kda_oracle.h")]
    if not force and os.path.exists(LIB):
        if os.path.getmtime(LIB) >= max(os.path.getmtime(s) for s in srcs):
            return LIB
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
           "-ffp-contract=off", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True, cwd=HERE)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def build_mutant(mutant: int, out_dir: str) -> str:
    """Compile a deliberately wrong variant of the oracle (KDA_ORACLE_MUTANT=mutant) into
    out_dir.  Only the pin-sensitivity test uses these; they are never trusted."""
    out = os.path.join(out_dir, f"libkda_oracle_mutant{mutant}.so")
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
           "-ffp-contract=off", f"-DKDA_ORACLE_MUTANT={int(mutant)}", "-o", out, SRC, "-lm"]
    subprocess.run(cmd, check=True, cwd=HERE)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
